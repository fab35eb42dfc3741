"""Benchmark of the Token Radius Attention hot path on B200.

One step = one pass of the whole hot path on the Wan2.1-14B 720p-shaped
workload (grid 21x45x80, N = 75600 tokens, 40 heads, d = 128, bf16, 128x128
blocks, gamma = 0.3, vote 1): a dense warm-up call (tile-major permute of Q,
K, V; dense attention + entropy; entropy -> radius; fused mask -> CSR; inverse
permute of O), then 4 block-sparse calls that reuse the warm-up's CSR on
perturbed Q/K (permute, block-sparse attention, inverse permute).  tau is
calibrated once (outside the timed region) so that ~12% of the blocks are kept.

`value` is the step's attention work on kept blocks (4*d*|qb|*|kb| flops per
kept block pair; the dense call keeps every pair) divided by the step time,
measured with CUDA events, inputs resident in HBM (each input tensor is
774 MB, larger than the 126 MB L2).  Per-kernel times come from CUDA events
around each launch on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun every rank runs its own independent workload (weak scaling:
different inputs, same shape; no collective on the data path).
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from entropy_adaptive_radius_b200 import inputs, workloads  # noqa: E402
from entropy_adaptive_radius_b200.pipeline import (Pipeline, calibrate_tau, full_csr,  # noqa: E402,F401
                                                   kept_pair_tokens)

METRIC = "block-sparse TRA attention ms/call & TFLOP/s (kept blocks) at 1 B200; mask ms"
UNIT = "TFLOP/s"
WL = workloads.WAN14B


# --------------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, path):
        self.index, self.path, self.proc = index, path, None

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons)}
        # median over the samples taken under load (top 80% of the clock samples)
        sm_sorted = sorted(sm)
        loaded = sm_sorted[len(sm_sorted) // 5:] or sm_sorted
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def sum_over_ranks(value, device=None):
    """Sum of a per-rank value over all ranks of the default process group
    (the value itself without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(value_ms, device=None):
    """Largest value over all ranks of the default process group (each rank
    times its own work with CUDA events; the job is as slow as its slowest
    rank).  Returns the value unchanged without a process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value_ms
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(wl, world):
    """The `config` object of the JSON line, identical in both arms: the
    workload's definition (shape, blocks, tile, gamma, vote threshold and the
    kept-block target tau is calibrated to).  Measured results (tau, kept
    fraction) are top-level keys of the line."""
    return {"workload": wl.name, "grid": [wl.F, wl.H, wl.W], "N": wl.N, "heads": wl.heads,
            "head_dim": wl.d, "block": [wl.block_q, wl.block_k], "tile": list(wl.tile),
            "gamma": wl.gamma, "vote": wl.vote, "kept_target": wl.kept_target,
            "sparse_calls_per_warmup": wl.sparse_calls, "l2": l2_note(wl),
            "parallelism": f"independent x{world}"}


# ------------------------------------------------------------------- GPU arm

WORKLOADS = {"wan14b": workloads.WAN14B, "wan13b": workloads.WAN13B,
             "hunyuan": workloads.HUNYUAN, "tiny": workloads.TINY}


def l2_note(wl):
    mb = wl.heads * wl.N * wl.d * 2 / 1e6
    if mb > 126:
        return f"inputs larger than L2 ({mb:.0f} MB per tensor)"
    return f"inputs fit in L2 ({mb:.1f} MB per tensor); L2 not flushed"


def time_ms(fn, reps=5, flush=None):
    """Median CUDA-event time of `fn` over `reps` launches after one untimed
    launch; `flush` (if given) runs before each timed launch, outside the
    events (an L2 flush)."""
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        ts.append(s.elapsed_time(e))
    return statistics.median(ts)


def time_ms_for(fn, seconds, flush=None):
    """time_ms over as many launches as fill about `seconds` of device time
    (at least 5): a kernel run back to back that long is in the power-capped
    steady state the measured sustained peak was taken in."""
    est = time_ms(fn, 1, flush)
    reps = int(max(5, min(2000, seconds * 1e3 / max(est, 1e-3))))
    return time_ms(fn, reps, flush)


def code_sha256(path):
    """sha256 of a C++/CUDA source with comments and whitespace removed: it
    changes when the code changes, not when only its comments do."""
    import hashlib
    import re
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return hashlib.sha256(re.sub(r"\s+", " ", src).strip().encode()).hexdigest()


def measured_traffic(wl, kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu capture of this
    workload, or None when there is none or the kernel code has changed since
    it was taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_wan14b.txt")
    if wl.name != workloads.WAN14B.name or not os.path.exists(path):
        return None
    rec = json.load(open(path))
    if code_sha256(os.path.join(ROOT, rec["source"])) != rec["source_code_sha256"] or kernel not in rec:
        return None
    return rec[kernel]["traffic_bytes"]


def entropy_overhead_ms(pipe, wl, device, pairs=5):
    """Cost of the entropy term of the dense warm-up call, measured apart from
    the step: dense attention with entropy (the warm-up kernel) and without it
    (the block-sparse kernel over a CSR that keeps every 128 x 128 block, the
    dense call's own tiling) are timed back to back `pairs` times, so both see
    the same clocks under the power cap; returns the medians of the plain time,
    the entropy-call time and their per-pair difference."""
    rp, ci = full_csr(wl.heads, wl.N, 128, device)
    t = pipe.tra
    dense = lambda: t.tra_dense_attn_entropy(pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm, pipe.H)  # noqa: E731
    plain = lambda: t.tra_block_sparse_attn(pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm, rp, ci,  # noqa: E731
                                            128, 128)
    dense()
    plain()
    torch.cuda.synchronize()
    d_ms, p_ms = [], []
    for i in range(pairs):
        for fn, acc in ((dense, d_ms), (plain, p_ms)) if i % 2 == 0 else ((plain, p_ms), (dense, d_ms)):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            torch.cuda.synchronize()
            acc.append(s.elapsed_time(e))
    diff = [a - b for a, b in zip(d_ms, p_ms)]
    return statistics.median(p_ms), statistics.median(d_ms), statistics.median(diff)


def gpu_arm(args, rank, world, local):
    import torch.distributed as dist
    from entropy_adaptive_radius_b200 import tra
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    log = (lambda m: print(f"[bench] {m}", file=sys.stderr, flush=True)) if rank == 0 else (lambda m: None)
    if world > 1:
        # short enough that ranks waiting on a lost rank fail soon; the longest
        # gap between two collectives here is well under a minute
        dist.init_process_group("nccl", device_id=device,
                                timeout=__import__("datetime").timedelta(seconds=180))
    wl = WORKLOADS[args.workload]
    calls = wl.sparse_calls
    t0 = time.time()
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, wl.dtype,
                              head_offset=rank * wl.heads)
    pert = [(inputs.perturb(Q, wl.seed, c, 0, head_offset=rank * wl.heads),
             inputs.perturb(K, wl.seed, c, 1, head_offset=rank * wl.heads)) for c in range(1, calls + 1)]
    log(f"inputs generated in {time.time() - t0:.1f}s")
    host = [Q, K, V] + [x for qk in pert for x in qk]
    # pinned copies replace the pageable ones (about 8.5 GB per rank at the
    # 14B shape, so a node running one rank per GPU holds one copy, not two)
    host = [x.pin_memory() for x in host]
    Q, K, V = host[0], host[1], host[2]
    del pert
    dev = [x.to(device) for x in host]
    Qd, Kd, Vd = dev[0], dev[1], dev[2]
    sparse_in = [(dev[3 + 2 * i], dev[4 + 2 * i], Vd) for i in range(calls)]

    pipe = Pipeline(wl, device)
    # dense warm-up once to get H, then calibrate tau on it
    pipe.warmup_call(Qd, Kd, Vd, None)
    torch.cuda.synchronize()
    pipe.tau = calibrate_tau(pipe, wl.kept_target, log) if wl.kept_target else wl.tau
    pipe.warmup_call(Qd, Kd, Vd, None)
    torch.cuda.synchronize()
    kept = pipe.kept_fraction()
    rp = pipe.row_ptr.cpu().numpy()
    ci = pipe.col_idx[: int(pipe.nnz.item())].cpu().numpy()
    kept_pairs = kept_pair_tokens(rp, ci, wl.heads, wl.N, wl.block_q, wl.block_k)
    fl_sparse = 4.0 * wl.d * kept_pairs                  # per sparse call
    fl_dense = 4.0 * wl.d * wl.N * wl.N * wl.heads      # the warm-up keeps every pair
    fl_step = fl_dense + calls * fl_sparse

    def step(rec):
        pipe.warmup_call(Qd, Kd, Vd, rec)
        for c in range(calls):
            pipe.sparse_call(*sparse_in[c], rec)

    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize()
    if tra.tra_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    clocks_csv = (args.clocks_csv.replace("{rank}", str(rank)) if args.clocks_csv
                  else os.path.join(tempfile.gettempdir(), f"tra_clocks_rank{rank}_{os.getpid()}.csv"))
    sampler = ClockSampler(local, clocks_csv)
    rec = []
    pipe.launches = 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    start.record()
    for _ in range(args.steps):
        step(rec)
    stop.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = start.elapsed_time(stop)
    launches = pipe.launches
    if world > 1:
        elapsed_ms = max_over_ranks(elapsed_ms, device)
        dist.barrier()
    if tra.tra_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out in the timed region")

    # entropy-overhead term: dense with and without entropy, interleaved
    plain_ms, dense_pair_ms, entropy_ms = entropy_overhead_ms(pipe, wl, device)

    # the same step with the tokens kept in tile-major order between calls (a
    # model that permutes once per transformer block): inputs permuted once,
    # outside the timed region; no permutes inside it
    def to_tm(X):
        Y = torch.empty(X.shape, dtype=torch.bfloat16, device=device)
        tra.tra_tile_major_permute(X, Y, pipe.grid, wl.tile)
        return Y
    res_main = [to_tm(X) for X in (Qd, Kd, Vd)]
    res_sparse = [(to_tm(q), to_tm(k), res_main[2]) for q, k, _ in sparse_in]
    res_out = torch.empty_like(pipe.O)

    def step_resident():
        pipe.warmup_call(*res_main, None, out=res_out, resident=True)
        for c in range(calls):
            pipe.sparse_call(*res_sparse[c], None, out=res_out, resident=True)

    step_resident()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    r_steps = max(1, min(args.steps, 3))
    rs, re_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rs.record()
    for _ in range(r_steps):
        step_resident()
    re_.record()
    torch.cuda.synchronize()
    res_ms = rs.elapsed_time(re_) / r_steps
    if world > 1:
        res_ms = max_over_ranks(res_ms, device)
    del res_main, res_sparse, res_out

    # per-kernel times (launching stream = current stream)
    dense_ms, sparse_ms, mask_ms, radius_ms, perm_ms = [], [], [], [], []
    for kind, e in rec:
        if kind == "warmup":
            perm_ms.append(e[0].elapsed_time(e[1]) + e[4].elapsed_time(e[5]))
            dense_ms.append(e[1].elapsed_time(e[2]))
            radius_ms.append(e[2].elapsed_time(e[3]))
            mask_ms.append(e[3].elapsed_time(e[4]))
        else:
            perm_ms.append(e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]))
            sparse_ms.append(e[1].elapsed_time(e[2]))
    ms_step = elapsed_ms / args.steps
    # whole-job work: every rank calibrates its own tau on its own inputs, so
    # the ranks' kept work differs a little; the job's flops are their sum
    fl_job = sum_over_ranks(fl_step, device) if world > 1 else fl_step
    value = fl_job / (ms_step * 1e-3) / 1e12
    d_ms, s_ms = statistics.mean(dense_ms), statistics.mean(sparse_ms)
    peaks, peak_kind = load_peaks()
    dense_tf = fl_dense / (d_ms * 1e-3) / 1e12
    sparse_tf = fl_sparse / (s_ms * 1e-3) / 1e12
    # dominant kernel of the step by device time
    dense_total, sparse_total = d_ms, calls * s_ms
    dom = ("dense_attn_entropy", dense_tf) if dense_total >= sparse_total else ("block_sparse_attn", sparse_tf)
    peak_sus = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    traffic = measured_traffic(wl, dom[0])
    roofline = {"kernel": dom[0], "bound": "tensor", "achieved": round(dom[1], 2),
                "peak": peak_sus, "unit": "TFLOP/s", "frac": round(dom[1] / peak_sus, 4),
                "traffic": traffic, "traffic_unit": "bytes per launch (ncu dram read + write)",
                "peak_kind": f"{peak_kind} bf16 sustained"}
    roofline_sparse = {"kernel": "block_sparse_attn", "bound": "tensor", "achieved": round(sparse_tf, 2),
                       "peak": peak_sus, "unit": "TFLOP/s", "frac": round(sparse_tf / peak_sus, 4)}
    hbm = peaks.get("hbm_gbs")
    perm_bytes = 2 * wl.heads * wl.N * wl.d * 2      # read + write of one tensor
    perm_per_launch_ms = statistics.mean(perm_ms) / 4.0  # 4 permute launches per call
    roofline_permute = {"kernel": "tile_major_permute", "bound": "hbm",
                        "achieved": round(perm_bytes / (perm_per_launch_ms * 1e-3) / 1e9, 1),
                        "peak": hbm, "unit": "GB/s",
                        "frac": round(perm_bytes / (perm_per_launch_ms * 1e-3) / 1e9 / hbm, 4)}
    mask_total = statistics.mean(mask_ms) + statistics.mean(radius_ms)
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Fourier-feature Q/K of grid position + noise, v ~ N(0,1))",
        "config": workload_config(wl, world),
        "tau": round(pipe.tau, 8), "kept_fraction": round(kept, 4),
        "sparse_ms_per_call": round(s_ms, 3), "sparse_tflops_kept": round(sparse_tf, 2),
        "dense_ms_per_call": round(d_ms, 3), "dense_tflops": round(dense_tf, 2),
        "mask_ms": round(statistics.mean(mask_ms), 3), "radius_ms": round(statistics.mean(radius_ms), 4),
        "permute_ms_per_call": round(statistics.mean(perm_ms), 3),
        "overhead_vs_sparse": {
            "entropy_ms": round(entropy_ms, 3), "plain_dense_ms": round(plain_ms, 3),
            "dense_entropy_ms_paired": round(dense_pair_ms, 3),
            "mask_plus_radius_ms": round(mask_total, 3),
            "total_ms": round(max(0.0, entropy_ms) + mask_total, 3),
            "ratio_to_sparse_calls": round((max(0.0, entropy_ms) + mask_total) / (calls * s_ms), 4),
            "unamortised_ratio_to_1_call": round((max(0.0, entropy_ms) + mask_total) / s_ms, 4),
            "sparse_calls": calls},
        "tile_major_resident": {"ms_per_step": round(res_ms, 3),
                                "value": round(fl_job / (res_ms * 1e-3) / 1e12, 3),
                                "unit": UNIT, "note": "same step, tokens kept in tile-major order "
                                "between calls: no per-call permutes"},
        "roofline": roofline, "roofline_sparse": roofline_sparse, "roofline_permute": roofline_permute,
        "clocks": clocks, "gpu_launches": launches,
    }

    # ---- end to end: host (pinned) inputs copied in, O copied back, every call
    e2e = e2e_run(pipe, host, dev, calls, args, device, world)
    out["e2e"] = {"value": round(fl_job / (e2e["ms"] * 1e-3) / 1e12, 3), "unit": UNIT,
                  "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                  "ms_per_step": round(e2e["ms"], 3)}
    if rank == 0 and world == 1:
        out["cpu_baseline"] = cpu_baseline(args, Q, K, V, pipe, kept_pairs, fl_step, wl)
    if world == 1 and wl is workloads.WAN14B and not args.no_configs:
        del pipe, dev, sparse_in, Qd, Kd, Vd, e2e
        torch.cuda.empty_cache()
        out["configs"] = other_configs(device, log)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def l2_flusher(device):
    """Writes a 256 MB buffer (twice the 126 MB L2) so the next launch starts
    with a cold L2."""
    buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    return lambda: buf.fill_(1)


def executed_over_kept(row_ptr, col_idx, heads, N, bq, bk):
    """Work the attention kernel executes over the kept work: with 64-token
    query blocks a 128-row tile runs the ascending union of its two blocks'
    key-block lists for all of its rows; otherwise 1."""
    if bq >= 128:
        return 1.0
    nqb = -(-N // bq)
    rp = row_ptr.reshape(heads, nqb + 1)
    ksz = np.minimum(bk, N - np.arange(-(-N // bk)) * bk).astype(np.int64)
    qsz = np.minimum(bq, N - np.arange(nqb) * bq).astype(np.int64)
    executed = kept = 0
    for h in range(heads):
        for t in range(0, nqb, 128 // bq):
            blocks = range(t, min(nqb, t + 128 // bq))
            cols = [col_idx[rp[h, b]:rp[h, b + 1]] for b in blocks]
            union = np.unique(np.concatenate(cols)) if cols else np.zeros(0, np.int64)
            executed += int(sum(qsz[b] for b in blocks)) * int(ksz[union].sum())
            kept += sum(int(qsz[b]) * int(ksz[c].sum()) for b, c in zip(blocks, cols))
    return executed / max(1, kept)


def config_point(wl, device, log, peak, flush):
    """One workload timed in the bench's run: dense warm-up (dense + entropy)
    call, tau calibrated to the kept target, then the block-sparse call over
    that CSR, the radius + mask, and (for one sparse call per warm-up) the
    unamortised entropy + mask overhead.  The attention kernels are timed back
    to back for about a second each (CUDA events per launch, median, L2
    flushed before each launch), the mask over 5 launches."""
    from entropy_adaptive_radius_b200 import tra
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, wl.dtype)
    Qd, Kd, Vd = Q.to(device), K.to(device), V.to(device)
    pipe = Pipeline(wl, device)
    pipe.warmup_call(Qd, Kd, Vd, None)
    pipe.tau = calibrate_tau(pipe, wl.kept_target, log)
    pipe.warmup_call(Qd, Kd, Vd, None)
    torch.cuda.synchronize()
    kept = pipe.kept_fraction()
    rp = pipe.row_ptr.cpu().numpy()
    ci = pipe.col_idx[: int(pipe.nnz.item())].cpu().numpy()
    pairs = kept_pair_tokens(rp, ci, wl.heads, wl.N, wl.block_q, wl.block_k)
    q, k, v, o = pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm
    sparse_ms = time_ms_for(lambda: tra.tra_block_sparse_attn(q, k, v, o, pipe.row_ptr,
                                                              pipe.col_idx, wl.block_q,
                                                              wl.block_k), 1.0, flush)
    dense_ms = time_ms_for(lambda: tra.tra_dense_attn_entropy(q, k, v, o, pipe.H), 1.0, flush)
    tau = pipe.tau
    mask_ms = time_ms(lambda: pipe.mask(tau), 5, flush)
    if tra.tra_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out")
    sparse_tf = 4.0 * wl.d * pairs / (sparse_ms * 1e-3) / 1e12
    dense_tf = 4.0 * wl.d * wl.N * wl.N * wl.heads / (dense_ms * 1e-3) / 1e12
    cfg = dict(workload_config(wl, 1), l2="L2 flushed before each timed launch")
    row = {"workload": wl.name, "config": cfg, "tau": round(tau, 8),
           "kept_fraction": round(kept, 4), "sparse_ms": round(sparse_ms, 3),
           "sparse_tflops_kept": round(sparse_tf, 1), "sparse_frac": round(sparse_tf / peak, 4),
           "executed_over_kept": round(executed_over_kept(rp, ci, wl.heads, wl.N, wl.block_q,
                                                          wl.block_k), 3),
           "dense_entropy_ms": round(dense_ms, 3), "dense_tflops": round(dense_tf, 1),
           "dense_frac": round(dense_tf / peak, 4), "mask_plus_radius_ms": round(mask_ms, 3)}
    if wl.block_q == 128:
        plain_ms, _, entropy_ms = entropy_overhead_ms(pipe, wl, device, pairs=3)
        over = max(0.0, entropy_ms) + mask_ms
        row["entropy_ms"] = round(entropy_ms, 3)
        row["overhead_ratio_to_sparse_calls"] = round(over / (wl.sparse_calls * sparse_ms), 4)
    del pipe, Qd, Kd, Vd
    torch.cuda.empty_cache()
    return row


def sweep_points(device, log, peak, flush, votes, targets):
    """The density sweep at the 21x45x80, 40-head shape on its own inputs:
    per vote threshold and target kept fraction, tau calibrated on the
    warm-up's entropy, then the block-sparse call (back to back for about half
    a second) and the radius + mask timed, L2 flushed before each launch; the
    100% point is the dense call."""
    from entropy_adaptive_radius_b200 import tra
    wl = workloads.SWEEP
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, wl.dtype)
    Qd, Kd, Vd = Q.to(device), K.to(device), V.to(device)
    pipe = Pipeline(wl, device)
    pipe.warmup_call(Qd, Kd, Vd, None)
    torch.cuda.synchronize()
    q, k, v, o = pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm
    dense_ms = time_ms_for(lambda: tra.tra_dense_attn_entropy(q, k, v, o, pipe.H), 1.0, flush)
    dense_tf = 4.0 * wl.d * wl.N * wl.N * wl.heads / (dense_ms * 1e-3) / 1e12
    points = []
    for vote in votes:
        pipe.vote = vote
        pipe.mask(1e-12)  # r ~ 0: the kept fraction's floor at this vote threshold
        floor = round(pipe.kept_fraction(), 4)
        for target in targets:
            if target >= 1.0:
                points.append({"vote": vote, "target_kept": 1.0, "kept_fraction": 1.0,
                               "kept_floor": floor, "path": "dense", "ms": round(dense_ms, 3),
                               "tflops_kept": round(dense_tf, 1),
                               "frac": round(dense_tf / peak, 4)})
                continue
            tau = calibrate_tau(pipe, target, log)
            pipe.mask(tau)
            torch.cuda.synchronize()
            rp = pipe.row_ptr.cpu().numpy()
            ci = pipe.col_idx[: int(pipe.nnz.item())].cpu().numpy()
            pairs = kept_pair_tokens(rp, ci, wl.heads, wl.N, wl.block_q, wl.block_k)
            ms = time_ms_for(lambda: tra.tra_block_sparse_attn(q, k, v, o, pipe.row_ptr,
                                                               pipe.col_idx, wl.block_q,
                                                               wl.block_k), 0.5, flush)
            mask_ms = time_ms(lambda: pipe.mask(tau), 3, flush)
            tf = 4.0 * wl.d * pairs / (ms * 1e-3) / 1e12
            points.append({"vote": vote, "target_kept": target,
                           "kept_fraction": round(pipe.kept_fraction(), 4), "kept_floor": floor,
                           "tau": round(tau, 8),
                           "path": "sparse", "ms": round(ms, 3), "tflops_kept": round(tf, 1),
                           "frac": round(tf / peak, 4), "speedup_vs_dense": round(dense_ms / ms, 2),
                           "mask_plus_radius_ms": round(mask_ms, 3)})
    if tra.tra_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out")
    del pipe, Qd, Kd, Vd
    torch.cuda.empty_cache()
    return {"workload": wl.name,
            "config": dict(workload_config(wl, 1), l2="L2 flushed before each timed launch"),
            "points": points}


def other_configs(device, log):
    """The other workloads, timed in the same run as the headline step: the
    Wan2.1-1.3B and HunyuanVideo-13B shapes and the density sweep."""
    peaks, kind = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    flush = l2_flusher(device)
    t0 = time.time()
    out = {"peak": f"{peak} TFLOP/s ({kind} bf16 sustained)",
           "timing": "attention kernels back to back for about 0.5-1 s each (the sustained peak's "
                     "method), mask over 3-5 launches; CUDA events per launch, median, L2 flushed "
                     "before each launch"}
    for key, wl in (("wan13b", workloads.WAN13B), ("hunyuan", workloads.HUNYUAN)):
        out[key] = config_point(wl, device, log, peak, flush)
        log(f"config {key} done ({time.time() - t0:.0f}s)")
    out["sweep"] = sweep_points(device, log, peak, flush, workloads.SWEEP.sweep_votes,
                                workloads.SWEEP.sweep)
    log(f"configs done ({time.time() - t0:.0f}s)")
    return out


def e2e_run(pipe, host, dev, calls, args, device, world):
    """End to end through the C ABI from pinned host memory.  Every step's
    inputs (its distinct tensors: Q, K, V of the warm-up call and Q_c, K_c of
    each sparse call, V being shared, all in the original token order) are
    copied host -> device, and every call's output O device -> host, inside
    the timed region.  Inputs are double-buffered per step on a copy-in
    stream, so the next step's inputs move while this step computes; outputs
    go back on a copy-out stream (the two directions run at once)."""
    comp = torch.cuda.current_stream(device)
    cin, cout = torch.cuda.Stream(device), torch.cuda.Stream(device)
    n_in = len(host)                        # 3 + 2 * calls distinct inputs
    sets = [[torch.empty_like(dev[i]) for i in range(n_in)] for _ in range(2)]
    outs = [[torch.empty_like(pipe.O) for _ in range(calls + 1)] for _ in range(2)]
    out_host = [torch.empty(pipe.O.shape, dtype=pipe.O.dtype).pin_memory() for _ in range(calls + 1)]
    ready = [[torch.cuda.Event() for _ in range(calls + 1)] for _ in range(2)]
    copied = [[torch.cuda.Event() for _ in range(calls + 1)] for _ in range(2)]
    step_done = [torch.cuda.Event(), torch.cuda.Event()]
    used = [False, False]
    # inputs of call c: (Q, K, V) for the warm-up, (Q_c, K_c, V) after it
    call_in = [(0, 1, 2)] + [(3 + 2 * c, 4 + 2 * c, 2) for c in range(calls)]
    nbytes_in = sum(x.numel() * x.element_size() for x in host)
    nbytes_out = (calls + 1) * out_host[0].numel() * out_host[0].element_size()

    def copy_in(st):
        with torch.cuda.stream(cin):
            if used[st]:
                cin.wait_event(step_done[st])   # the step that last used this set is done
            done = set()
            for c, idx in enumerate(call_in):
                for i in idx:
                    if i not in done:
                        sets[st][i].copy_(host[i], non_blocking=True)
                        done.add(i)
                ready[st][c].record(cin)

    def compute(st):
        for c, (iq, ik, iv) in enumerate(call_in):
            comp.wait_event(ready[st][c])
            if used[st]:
                comp.wait_event(copied[st][c])  # this output buffer has been read back
            q, k, v = sets[st][iq], sets[st][ik], sets[st][iv]
            if c == 0:
                pipe.warmup_call(q, k, v, None, out=outs[st][c])
            else:
                pipe.sparse_call(q, k, v, None, out=outs[st][c])
            ev = torch.cuda.Event()
            ev.record(comp)
            with torch.cuda.stream(cout):
                cout.wait_event(ev)
                out_host[c].copy_(outs[st][c], non_blocking=True)
                copied[st][c].record(cout)
        step_done[st].record(comp)
        used[st] = True

    def run(n):
        copy_in(0)
        for k in range(n):
            if k + 1 < n:
                copy_in((k + 1) % 2)
            compute(k % 2)
        comp.wait_stream(cout)

    run(2)   # warm-up
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    steps = max(2, min(args.steps, 4))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    run(steps)
    e.record(comp)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e)
    if world > 1:
        ms = max_over_ranks(ms, device)
    return {"ms": ms / steps, "h2d": nbytes_in, "d2h": nbytes_out}


# ------------------------------------------------------------- CPU baselines

def oracle_throughput(Q, K, V, wl, tau, kept_frac):
    """The oracle (as it stands) on a bounded sample of one step's work: dense
    attention + entropy rows, radius for all queries of one head, brute-force
    mask rows, sparse attention rows.  Returns the extrapolated step time (s)
    and what was sampled."""
    from oracle import tra_oracle as O
    N, d = wl.N, wl.d
    scale = 1.0 / math.sqrt(d)
    grid = (wl.F, wl.H, wl.W)
    pi = O.tile_major_order(*grid, wl.tile)
    c = O.token_coords(*grid)[pi]
    q = O.permute(Q[0:1].double().numpy(), pi)[0]
    k = O.permute(K[0:1].double().numpy(), pi)[0]
    v = O.permute(V[0:1].double().numpy(), pi)[0]
    rows = np.arange(0, min(256, N))
    t0 = time.perf_counter()
    _, Hs, _ = O.attention_rows(q, k, v, scale, rows)
    t_dense_row = (time.perf_counter() - t0) / len(rows)
    # radius of every query of one head (entropy stand-in: the sampled values tiled)
    Hfull = np.resize(Hs, N)
    t0 = time.perf_counter()
    r = O.radius(Hfull, c[:, 2], tau, wl.gamma, wl.F, N).astype(np.float32)
    t_radius_head = time.perf_counter() - t0
    phi32 = O.phi(np.arange(wl.F), wl.gamma).astype(np.float32)
    t0 = time.perf_counter()
    bm = O.block_mask(r, phi32, c, wl.block_q, wl.block_k, wl.vote, qblocks=[0, min(1, wl.nqb - 1)])
    t_mask_row = (time.perf_counter() - t0) / 2
    nkb = wl.nkb
    mrow = np.zeros((wl.nqb, nkb), bool)
    mrow[0] = bm[0]
    mrow[1] = bm[1]
    t0 = time.perf_counter()
    O.sparse_attention_rows(q, k, v, mrow, wl.block_q, wl.block_k, scale, rows)
    t_sparse_row_measured = (time.perf_counter() - t0) / len(rows)
    # the oracle's sparse row costs like a dense row over the kept keys; scale the
    # measured row (kept fraction of its own rows) to the workload's kept fraction
    own = max(1e-9, float(bm.mean()))
    t_sparse_row = t_sparse_row_measured * kept_frac / own if own > 0 else t_sparse_row_measured
    heads = wl.heads
    t_step = (heads * N * t_dense_row + heads * t_radius_head + heads * wl.nqb * t_mask_row
              + wl.sparse_calls * heads * N * t_sparse_row)
    sample = (f"one head: 256 dense+entropy rows, radius of all {N} queries, 2 brute-force mask "
              f"block rows, 256 sparse rows; extrapolated to {heads} heads x (1 dense + "
              f"{wl.sparse_calls} sparse calls)")
    return t_step, sample


def host_threads():
    """Threads the oracle's numpy/BLAS calls actually use."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(args, Q, K, V, pipe, kept_pairs, fl_step, wl):
    kept_frac = kept_pairs / (wl.heads * wl.N * wl.N)
    t_step, sample = oracle_throughput(Q, K, V, wl, pipe.tau, kept_frac)
    return {"value": round(fl_step / t_step / 1e12, 6), "unit": UNIT,
            "cores": host_threads(), "kind": "oracle", "sample": sample,
            "extrapolated_step_s": round(t_step, 1)}


def sweep_arm(args):
    """Density sweep at the 21x45x80, 40-head shape on its own inputs (the
    points the default line carries under `configs.sweep`): for each vote
    threshold and target kept fraction, tau is bisected to the target (or the
    nearest reachable fraction: every query keeps its own position in every
    frame, so the fraction has a floor), then the block-sparse call and the
    radius + mask are timed against the dense call.  One JSON line per point."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    log = lambda m: print(f"[sweep] {m}", file=sys.stderr, flush=True)  # noqa: E731
    peaks, kind = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    wl = workloads.SWEEP
    res = sweep_points(device, log, peak, l2_flusher(device), wl.sweep_votes, wl.sweep)
    for point in res["points"]:
        print(json.dumps(dict(workload=res["workload"], peak=f"{peak} TFLOP/s ({kind} bf16 sustained)",
                              **point)), flush=True)


def variants_arm(args):
    """Mask variants at the 21x45x80, 40-head shape: TRA's per-query entropy
    budget with the disk, the shared per-head budget (entropy mapping removed),
    the 1D distance, and Radial Attention's static window (disk and 1D).  Each
    variant's parameter (tau, or r0 for Radial) is bisected to the same kept
    fraction as the bench's TRA workload; then its radius + mask time and the
    block-sparse call over its CSR are timed.  One JSON line per variant."""
    from entropy_adaptive_radius_b200 import tra
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = workloads.WAN14B
    log = lambda m: print(f"[variants] {m}", file=sys.stderr, flush=True)  # noqa: E731
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, wl.dtype)
    Qd, Kd, Vd = Q.to(device), K.to(device), V.to(device)
    pipe = Pipeline(wl, device)
    pipe.warmup_call(Qd, Kd, Vd, None)
    torch.cuda.synchronize()
    peaks, kind = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    for source, metric in (("entropy", "disk"), ("shared", "disk"), ("entropy", "line"),
                           ("radial", "disk"), ("radial", "line")):
        pipe.variant = (source, metric)
        param = calibrate_tau(pipe, wl.kept_target, log)
        pipe.mask(param)
        kept = pipe.kept_fraction()
        rp = pipe.row_ptr.cpu().numpy()
        ci = pipe.col_idx[: int(pipe.nnz.item())].cpu().numpy()
        pairs = kept_pair_tokens(rp, ci, wl.heads, wl.N, wl.block_q, wl.block_k)
        ms = time_ms(lambda: tra.tra_block_sparse_attn(
            pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm, pipe.row_ptr, pipe.col_idx,
            wl.block_q, wl.block_k), 5)
        radius_ms = time_ms(lambda: pipe.radius(param), 5)
        mask_ms = time_ms(lambda: pipe.mask(param), 5)
        if tra.tra_get_device_error() != 0:
            raise RuntimeError("device-side wait timed out")
        tf = 4.0 * wl.d * pairs / (ms * 1e-3) / 1e12
        print(json.dumps({
            "workload": wl.name, "variant": {"budget": source, "metric": metric},
            "param": {"r0" if source == "radial" else "tau": round(param, 8)},
            "kept_fraction": round(kept, 4), "radius_ms": round(radius_ms, 4),
            "radius_plus_mask_ms": round(mask_ms, 3), "sparse_ms": round(ms, 3),
            "sparse_tflops_kept": round(tf, 1), "roofline_frac": round(tf / peak, 4),
            "peak": f"{peak} TFLOP/s ({kind} bf16 sustained)"}), flush=True)


def reuse_arm(args):
    """Cross-step reuse at the 21x45x80, 40-head shape: a 50-step denoising
    run of one attention layer through the layer driver, for several reuse
    policies (all steps dense; one dense warm-up then sparse; and entropy
    refreshes every 10 steps, by an entropy-only pass or by a dense step).
    Inputs stay on the GPU (the step's Q, K cycle through five perturbed
    copies); each run is timed with CUDA events.  One JSON line per policy."""
    from entropy_adaptive_radius_b200 import tra
    from entropy_adaptive_radius_b200.layer import ReusePolicy, TraLayer
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = workloads.WAN14B
    log = lambda m: print(f"[reuse] {m}", file=sys.stderr, flush=True)  # noqa: E731
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, wl.dtype)
    seq = [(Q.to(device), K.to(device))]
    for c in range(1, 5):
        seq.append((inputs.perturb(Q, wl.seed, c, 0).to(device), inputs.perturb(K, wl.seed, c, 1).to(device)))
    Vd = V.to(device)
    pipe = Pipeline(wl, device)
    pipe.warmup_call(seq[0][0], seq[0][1], Vd, None)
    tau = calibrate_tau(pipe, wl.kept_target, log)
    del pipe
    steps = 50
    policies = [("all dense", ReusePolicy(warmup=steps)),
                ("warm-up 1, no refresh", ReusePolicy(warmup=1)),
                ("warm-up 1, entropy-only refresh every 10", ReusePolicy(1, 10, "entropy")),
                ("warm-up 1, dense refresh every 10", ReusePolicy(1, 10, "dense"))]
    O_ = torch.empty_like(Vd)
    # load every kernel once before any timing (the entropy-only one is first
    # needed mid-run by the refresh policies)
    tra.tra_attn_entropy(seq[0][0], seq[0][1],
                         torch.empty(wl.heads, wl.N, dtype=torch.float32, device=device))
    base = None
    for name, pol in policies:
        layer = TraLayer((wl.F, wl.H, wl.W), wl.heads, wl.d, tau=tau, gamma=wl.gamma, tile=wl.tile,
                         block_q=wl.block_q, block_k=wl.block_k, vote=wl.vote, policy=pol,
                         device=device)
        for k in range(3):   # warm the kernels once (dense, sparse and refresh kinds)
            layer(seq[0][0], seq[0][1], Vd, O_)
        layer.reset()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for k in range(steps):
            q, kk = seq[k % len(seq)]
            layer(q, kk, Vd, O_)
        e.record()
        torch.cuda.synchronize()
        if tra.tra_get_device_error() != 0:
            raise RuntimeError("device-side wait timed out")
        ms = s.elapsed_time(e)
        base = ms if base is None else base
        kinds = [pol.kind(k) for k in range(steps)]
        print(json.dumps({
            "workload": wl.name, "policy": name, "steps": steps,
            "dense_steps": kinds.count("dense"), "entropy_only_refreshes": kinds.count("sparse+entropy"),
            "tau": round(tau, 6), "kept_fraction_last_mask": round(int(layer.nnz.item()) / (wl.heads * layer.nqb * layer.nkb), 4),
            "ms_per_run": round(ms, 2), "ms_per_step": round(ms / steps, 3),
            "attention_speedup_vs_all_dense": round(base / ms, 3)}), flush=True)
        del layer


def reference_arm(args, rank, world):
    if rank != 0:
        return
    wl = WORKLOADS.get(args.workload, WL)
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, 1, wl.d, wl.seed, wl.q_scale, wl.dtype)
    kept = wl.kept_target if wl.kept_target else 1.0
    fl_sparse = 4.0 * wl.d * wl.N * wl.N * wl.heads * kept
    fl_step = 4.0 * wl.d * wl.N * wl.N * wl.heads + wl.sparse_calls * fl_sparse
    times, walls = [], []
    sample = ""
    for i in range(args.warmup + args.steps):
        w0 = time.perf_counter()
        t_step, sample = oracle_throughput(Q, K, V, wl, 0.01, kept)
        if i >= args.warmup:
            times.append(t_step)
            walls.append(time.perf_counter() - w0)
    t = statistics.mean(times)
    v = fl_step / t / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           # a step is the bounded sample; the rate is its cost extrapolated to
           # the whole step of the workload
           "ms_per_step": round(statistics.mean(walls) * 1e3, 1), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(wl, world),
           "tau": None, "kept_fraction": kept,
           "extrapolated_full_step_s": round(t, 1),
           "note": "each step is a bounded sample of the workload's step; the rate extrapolates "
                   "its cost to the whole step at the workload's kept-block target",
           "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": host_threads(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def kernel_case(args):
    """Small single-kernel cases for profiler captures (inputs > L2, < 1 GB):
    dense / sparse / entropy (entropy only, no PV) / sparse_fp8 (E4M3 Q, K) /
    quant (E4M3 quantization of Q): 40 heads x 16384 tokens x d=128 bf16
    (168 MB per tensor);
    sparse64: the Wan2.1-1.3B shape (12 x 32760 x 128, 64-token blocks) on its
    own radius mask at the calibrated kept fraction;
    sparse14b: the Wan2.1-14B shape (40 x 75600 x 128, 128-token blocks) on its
    own radius mask at the calibrated ~12% kept blocks;
    mask: the 21x45x80 grid, 40 heads, radii from entropies near ln N;
    permute: one 21x45x80 x 40-head x 128 bf16 tensor.  Runs the kernel
    `--reps` times and prints the mean CUDA-event time per launch."""
    from entropy_adaptive_radius_b200 import tra
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(0)
    heads, N, d = 40, 16384, 128
    reps = args.reps
    if args.case == "sparse14b":
        # the Wan2.1-14B shape with its own band mask at the calibrated ~12%
        # kept blocks; the original-order inputs and output are freed before
        # the timed launches (about 3.2 GB stays on the device: Q, K, V, O in
        # tile-major order, the entropy, radii and the CSR)
        wl = workloads.WAN14B
        Q, K, V = (t.to(dev) for t in inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed,
                                                      wl.q_scale, "bf16"))
        pipe = Pipeline(wl, dev)
        pipe.warmup_call(Q, K, V, None)
        pipe.mask(calibrate_tau(pipe, wl.kept_target, lambda m: print(f"[bench] {m}", file=sys.stderr)))
        torch.cuda.synchronize()
        del Q, K, V
        pipe.O = None
        torch.cuda.empty_cache()
        rp_h = pipe.row_ptr.cpu().numpy()
        ci_h = pipe.col_idx.cpu().numpy()
        flops = 4.0 * wl.d * kept_pair_tokens(rp_h, ci_h, wl.heads, wl.N, wl.block_q, wl.block_k)
        q, k, v, o = pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm
        fn = lambda: tra.tra_block_sparse_attn(q, k, v, o, pipe.row_ptr, pipe.col_idx,  # noqa: E731
                                               wl.block_q, wl.block_k)
        unit = ("TFLOP/s", flops / 1e12)
    elif args.case == "sparse64":
        # the Wan2.1-1.3B shape with its own radius mask (64-token blocks, so
        # each 128-row tile runs the union of two query blocks' rows)
        wl = workloads.WAN13B
        Q, K, V = (t.to(dev) for t in inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed,
                                                      wl.q_scale, "bf16"))
        pipe = Pipeline(wl, dev)
        pipe.warmup_call(Q, K, V, None)
        pipe.mask(calibrate_tau(pipe, wl.kept_target, lambda m: print(f"[bench] {m}", file=sys.stderr)))
        rp_h = pipe.row_ptr.cpu().numpy()
        ci_h = pipe.col_idx.cpu().numpy()
        flops = 4.0 * wl.d * kept_pair_tokens(rp_h, ci_h, wl.heads, wl.N, wl.block_q, wl.block_k)
        q, k, v, o = pipe.Qtm, pipe.Ktm, pipe.Vtm, pipe.Otm
        fn = lambda: tra.tra_block_sparse_attn(q, k, v, o, pipe.row_ptr, pipe.col_idx,  # noqa: E731
                                               wl.block_q, wl.block_k)
        unit = ("TFLOP/s", flops / 1e12)
    elif args.case in ("dense", "sparse", "sparse_fp8", "quant", "entropy"):
        Q = (torch.randn(heads, N, d, generator=g, device=dev) * 2).to(torch.bfloat16)
        K = torch.randn(heads, N, d, generator=g, device=dev).to(torch.bfloat16)
        V = torch.randn(heads, N, d, generator=g, device=dev).to(torch.bfloat16)
        O_ = torch.empty_like(Q)
        H = torch.empty(heads, N, dtype=torch.float32, device=dev)
        nb = N // 128
        mask = inputs.synthetic_block_mask(heads, nb, nb, seed=0, density=0.12)
        rp, ci = inputs.csr_from_block_mask(mask)
        rpd, cid = torch.from_numpy(rp.ravel()).to(dev), torch.from_numpy(ci).to(dev)
        kept = int(mask.sum()) * 128 * 128
        if args.case == "dense":
            fn = lambda: tra.tra_dense_attn_entropy(Q, K, V, O_, H)  # noqa: E731
            flops = 4.0 * d * N * N * heads
        elif args.case == "entropy":
            fn = lambda: tra.tra_attn_entropy(Q, K, H)  # noqa: E731
            flops = 2.0 * d * N * N * heads     # QK^T only
        elif args.case in ("sparse_fp8", "quant"):
            Q8 = torch.empty(heads, N, d, dtype=torch.uint8, device=dev)
            K8 = torch.empty_like(Q8)
            qs = torch.empty(heads, N // 128, dtype=torch.float32, device=dev)
            ks = torch.empty_like(qs)
            tra.tra_quantize_e4m3(Q, Q8, qs)
            tra.tra_quantize_e4m3(K, K8, ks)
            if args.case == "quant":
                fn = lambda: tra.tra_quantize_e4m3(Q, Q8, qs)  # noqa: E731
                unit = ("GB/s", heads * N * d * 3 / 1e9)    # 2 bytes read + 1 written per element
            else:
                fn = lambda: tra.tra_block_sparse_attn_fp8(Q8, qs, K8, ks, V, O_, rpd, cid)  # noqa: E731
                flops = 4.0 * d * kept
        else:
            fn = lambda: tra.tra_block_sparse_attn(Q, K, V, O_, rpd, cid, 128, 128)  # noqa: E731
            flops = 4.0 * d * kept
        if args.case != "quant":
            unit = ("TFLOP/s", flops / 1e12)
    elif args.case == "mask":
        wl = WL
        grid = (wl.F, wl.H, wl.W)
        Hs = inputs.synthetic_entropy(wl.heads, wl.N, 0, math.log(wl.N) - 2.0, math.log(wl.N))
        Hd = torch.from_numpy(Hs).to(dev)
        r = torch.empty_like(Hd)
        phi = torch.empty(wl.F, dtype=torch.float32, device=dev)
        tra.tra_budget_radius(Hd, r, grid, 0.05, wl.gamma, wl.tile, phi_out=phi)
        ws = tra.workspace_tensor(tra.tra_mask_workspace_size(wl.heads, grid, 128, 128, wl.tile), dev)
        rp = torch.empty(wl.heads * (wl.nqb + 1), dtype=torch.int32, device=dev)
        ci = torch.empty(wl.heads * wl.nqb * wl.nkb, dtype=torch.int32, device=dev)
        nnz = torch.empty(1, dtype=torch.int32, device=dev)
        fn = lambda: tra.tra_build_block_mask(r, phi, grid, 128, 128, args.vote, rp, ci, nnz, ws,  # noqa: E731
                                             wl.tile)
        unit = ("Gpairs/s", wl.heads * wl.N * wl.N / 1e9)
    else:
        wl = WL
        grid = (wl.F, wl.H, wl.W)
        X = torch.randn(wl.heads, wl.N, wl.d, generator=g, device=dev).to(torch.bfloat16)
        Y = torch.empty_like(X)
        fn = lambda: tra.tra_tile_major_permute(X, Y, grid, wl.tile)  # noqa: E731
        unit = ("GB/s", 2 * X.numel() * 2 / 1e9)
    fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    if tra.tra_get_device_error() != 0:
        raise RuntimeError("device-side wait timed out")
    ms = s.elapsed_time(e) / reps
    print(json.dumps({"case": args.case, "ms_per_launch": round(ms, 4),
                      "rate": round(unit[1] / (ms * 1e-3), 2), "unit": unit[0]}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=["dense", "sparse", "sparse14b", "sparse64", "sparse_fp8", "quant", "entropy", "mask",
                                       "permute"], default=None,
                    help="run one kernel on a small case (for profiler captures)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--vote", type=int, default=1, help="vote threshold of the mask case")
    ap.add_argument("--workload", default="wan14b", choices=sorted(WORKLOADS) + ["sweep", "variants", "reuse"],
                    help="wan14b (default, the headline step), wan13b, hunyuan, tiny, the "
                         "density sweep, the mask variants, or the reuse policies")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tra", choices=["tra", "reference"])
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' points (Wan2.1-1.3B, HunyuanVideo, the "
                         "density sweep) that the 1-GPU line carries under `configs`")
    ap.add_argument("--clocks-csv", default=None,
                    help="where the nvidia-smi clock samples of the timed region go "
                         "({rank} is replaced by the rank); default: a temporary file")
    args = ap.parse_args()
    rank, world, local = dist_env()
    if args.case is not None:
        kernel_case(args)
        return
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if args.workload == "sweep":
        sweep_arm(args)
        return
    if args.workload == "variants":
        variants_arm(args)
        return
    if args.workload == "reuse":
        reuse_arm(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    gpu_arm(args, rank, world, local)


if __name__ == "__main__":
    main()
