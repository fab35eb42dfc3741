"""Calls from several host threads on distinct streams (the C ABI allows it:
each call only reads its arguments and launches on its own stream; the
library's lazily filled caches are guarded).  Four threads each run the
chained path (permute -> dense + entropy -> radius -> mask -> block-sparse
attention -> inverse permute) on their own inputs and stream, three times
over; every output must equal, bit for bit, the same chain run alone on the
default stream (every kernel here is deterministic)."""
import threading

import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from entropy_adaptive_radius_b200.pipeline import Pipeline
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _workload(i):
    block = 128 if i % 2 == 0 else 64
    return workloads.Workload(name=f"thread{i}", F=4, H=12 + i, W=20, heads=3, d=128,
                              dtype="bf16", block_q=block, block_k=block, gamma=0.3,
                              vote=1 + i, seed=20 + i, tau=0.05, sparse_calls=1)


def _chain(wl, dev, Q, K, V):
    pipe = Pipeline(wl, dev)
    pipe.tau = wl.tau
    out_d = torch.empty_like(Q)
    lse_d = torch.empty(wl.heads, wl.N, dtype=torch.float32, device=dev)
    pipe.warmup_call(Q, K, V, None, out=out_d, lse=lse_d)
    out_s = torch.empty_like(Q)
    lse_s = torch.empty_like(lse_d)
    pipe.sparse_call(Q, K, V, None, out=out_s, lse=lse_s)
    n = pipe.nnz.clone()
    return dict(out_d=out_d, lse_d=lse_d, H=pipe.H.clone(), r=pipe.r.clone(),
                row_ptr=pipe.row_ptr.clone(), col_idx=pipe.col_idx.clone(), nnz=n,
                out_s=out_s, lse_s=lse_s)


def test_concurrent_threads_on_distinct_streams_match_serial_runs():
    need_gpu()
    dev = torch.device("cuda", 0)
    wls = [_workload(i) for i in range(4)]
    data = []
    for wl in wls:
        Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, "bf16")
        data.append(tuple(x.to(dev) for x in (Q, K, V)))
    torch.cuda.synchronize()
    ref = []
    for wl, (Q, K, V) in zip(wls, data):
        ref.append({k: v.cpu() for k, v in _chain(wl, dev, Q, K, V).items()})
    assert tra.tra_get_device_error() == 0

    results = [[None] * 3 for _ in wls]
    errors = []

    def worker(i):
        try:
            torch.cuda.set_device(dev)
            s = torch.cuda.Stream(device=dev)
            with torch.cuda.stream(s):
                for rep in range(3):
                    got = _chain(wls[i], dev, *data[i])
                    s.synchronize()
                    results[i][rep] = {k: v.cpu() for k, v in got.items()}
        except Exception as e:  # reported below, in the main thread
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(wls))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not errors, errors
    torch.cuda.synchronize()
    assert tra.tra_get_device_error() == 0
    for i, wl in enumerate(wls):
        n = int(ref[i]["nnz"].item())
        assert 0 < n
        for rep in range(3):
            got = results[i][rep]
            for k, v in ref[i].items():
                a, b = got[k], v
                if k == "col_idx":
                    a, b = a[:n], b[:n]
                assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                                   b.view(torch.int16) if b.dtype == torch.bfloat16 else b), \
                    (wl.name, rep, k)
