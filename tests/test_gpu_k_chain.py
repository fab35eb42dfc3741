"""Chained GPU parity: the whole path as the benchmark runs it,
through the package's Pipeline (Token Radius Attention summary, §2 "TRA
pipeline": entropy from one dense warm-up call -> budget -> radius -> fused
radius mask -> block-sparse attention over the kept blocks, reused by the
later calls on drifting inputs).

For each workload shaped like the summary's models (Wan2.1-1.3B, Wan2.1-14B
with 4 sparse calls on Q/K + 0.05 N(0,1) over the warm-up's CSR,
HunyuanVideo-13B, and the density sweep's seed at vote thresholds 1, 4 and
16), the chain runs on all heads, and the oracle checks seeded samples:

  * the warm-up's O (original token order, after the inverse permute), H and
    LSE on sampled query tiles (the first, a middle, the last partial one and
    a random one) of three heads, against fp64 attention of the
    oracle-permuted inputs;
  * every radius against the oracle's radius of the GPU's own entropy
    (2e-6 relative), and the sampled ones against the radius of the oracle's
    entropy (the 1e-3 entropy tolerance moves r by at most 5.0e-4 relative);
  * the CSR rows of the sampled query blocks, bit for bit, against the
    brute-force block mask of the GPU's own fp32 radii and decay table, and
    the whole CSR for validity;
  * every sparse call's O and LSE on the sampled rows, against fp64 sparse
    attention of that call's oracle-permuted inputs over those mask rows.

Three mid-size chains (N = 1430 .. 2064, ragged tiles and tails, d = 64 and
128, blocks of 64 and 128 tokens, vote thresholds 1, 4 and 16) are compared
with the oracle on every element instead of samples.

The chained check can only compare a stage with the oracle given the GPU's
own upstream result: an entropy within 1e-3 may move a radius across a token
distance, so masks are compared for identical fp32 radii, as the
bit-exactness target states.
"""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from entropy_adaptive_radius_b200.pipeline import Pipeline, calibrate_tau
from oracle import tra_oracle as O
from tests.gpu_util import (H_ABS, LSE_ABS, check_attention, check_close, check_csr_valid,
                            csr_rows, need_gpu, to64)

pytestmark = pytest.mark.gpu

# r ~ exp(H / 2): an entropy error of 1e-3 moves r by exp(5e-4) - 1 < 5.002e-4
R_FROM_ORACLE_H_RTOL = 5.1e-4


def sample(wl, seed):
    """Sampled heads and query blocks: three heads; whole 128-row tiles (two
    64-token query blocks each on the Wan2.1-1.3B shape): the first, a
    middle, the last (partial) and a random one."""
    rng = np.random.default_rng(1000 + seed)
    heads = sorted({0, wl.heads - 1, int(rng.integers(1, wl.heads - 1))})
    per_tile = 128 // wl.block_q
    ntiles = -(-wl.N // 128)
    tiles = sorted({0, ntiles // 2, ntiles - 1, int(rng.integers(1, ntiles - 1))})
    qbs = sorted({qb for t in tiles for qb in range(t * per_tile, min(wl.nqb, (t + 1) * per_tile))})
    rows = np.concatenate([np.arange(qb * wl.block_q, min(wl.N, (qb + 1) * wl.block_q))
                           for qb in qbs])
    return heads, qbs, rows


class Chain:
    """One workload's inputs on the device, its Pipeline and the oracle-side
    views (tile-major order pi and token coordinates)."""

    def __init__(self, wl):
        self.wl = wl
        self.dev = torch.device("cuda", 0)
        self.grid = (wl.F, wl.H, wl.W)
        self.Q, self.K, self.V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed,
                                                 wl.q_scale, wl.dtype)
        self.Qd, self.Kd, self.Vd = (X.to(self.dev) for X in (self.Q, self.K, self.V))
        self.pipe = Pipeline(wl, self.dev)
        self.pi = O.tile_major_order(*self.grid, wl.tile)
        self.c = O.token_coords(*self.grid)[self.pi]
        self.scale = 1.0 / math.sqrt(wl.d)
        self.heads, self.qbs, self.rows = sample(wl, wl.seed)
        self.orig_rows = torch.from_numpy(self.pi[self.rows]).to(self.dev)

    def warmup(self, tau):
        """Dense warm-up call at tau; returns its output and LSE."""
        p = self.pipe
        p.tau = tau
        out = torch.empty_like(self.Qd)
        lse = torch.empty(self.wl.heads, self.wl.N, dtype=torch.float32, device=self.dev)
        p.warmup_call(self.Qd, self.Kd, self.Vd, None, out=out, lse=lse)
        torch.cuda.synchronize()
        assert tra.tra_get_device_error() == 0
        return out, lse

    def sparse(self, Qd, Kd):
        out = torch.empty_like(self.Qd)
        lse = torch.empty(self.wl.heads, self.wl.N, dtype=torch.float32, device=self.dev)
        self.pipe.sparse_call(Qd, Kd, self.Vd, None, out=out, lse=lse)
        torch.cuda.synchronize()
        assert tra.tra_get_device_error() == 0
        return out, lse

    def tm(self, X, h):
        """Head h of X (original order, CPU) in tile-major order, float64."""
        return to64(X[h])[self.pi]

    def out_rows(self, out, h):
        """Sampled tile-major rows of an original-order output of head h."""
        return out[h].index_select(0, self.orig_rows)


def check_warmup(ch, out, lse):
    wl, p = ch.wl, ch.pipe
    Hg = to64(p.H)
    assert np.isfinite(Hg).all()
    assert (Hg <= math.log(wl.N) + H_ABS).all() and (Hg >= -H_ABS).all()
    for h in ch.heads:
        q, k, v = ch.tm(ch.Q, h), ch.tm(ch.K, h), ch.tm(ch.V, h)
        Or, Hr, Lr = O.attention_rows(q, k, v, ch.scale, ch.rows)
        check_attention(ch.out_rows(out, h), Or, f"{wl.name} warm-up O h{h}")
        check_close(Hg[h, ch.rows], Hr, H_ABS, f"{wl.name} H h{h}")
        check_close(to64(lse)[h, ch.rows], Lr, LSE_ABS, f"{wl.name} LSE h{h}")
        # radius of the oracle's own entropy, on the sampled rows
        r_ref = O.radius(Hr, ch.c[ch.rows, 2], float(np.float32(p.tau)),
                         float(np.float32(wl.gamma)), wl.F, wl.N)
        assert np.allclose(to64(p.r)[h, ch.rows], r_ref, rtol=R_FROM_ORACLE_H_RTOL, atol=0)


def check_radius_and_mask(ch, vote):
    """Radii of the GPU entropy, decay table, and the sampled CSR rows bit for
    bit against the brute-force mask of the GPU's fp32 radii; returns the
    oracle's mask rows of the sampled heads ([nqb, nkb] with only the sampled
    query blocks filled)."""
    wl, p = ch.wl, ch.pipe
    tau32, gamma32 = float(np.float32(p.tau)), float(np.float32(wl.gamma))
    Hg, rg = to64(p.H), p.r.cpu().numpy()
    phig = p.phi.cpu().numpy()
    assert np.allclose(phig, O.phi(np.arange(wl.F), gamma32), rtol=6e-8, atol=0)
    for h in range(wl.heads):
        assert np.allclose(rg[h], O.radius(Hg[h], ch.c[:, 2], tau32, gamma32, wl.F, wl.N),
                           rtol=2e-6, atol=0), f"radius h{h}"
    nnz = int(p.nnz.item())
    rp = p.row_ptr.cpu().numpy()
    ci = p.col_idx[:nnz].cpu().numpy()
    check_csr_valid(rp, ci, nnz, wl.heads, wl.nqb, wl.nkb)
    masks = {}
    for h in ch.heads:
        ref = O.block_mask(rg[h], phig, ch.c, wl.block_q, wl.block_k, vote, qblocks=ch.qbs)
        m = np.zeros((wl.nqb, wl.nkb), dtype=bool)
        for row, qb in enumerate(ch.qbs):
            got = csr_rows(rp, ci, h, qb, wl.nqb)
            assert np.array_equal(got, np.nonzero(ref[row])[0]), (wl.name, h, qb, vote)
            m[qb] = ref[row]
        masks[h] = m
    return masks


def check_sparse(ch, masks, out, lse, Qc, Kc, what):
    wl = ch.wl
    for h in ch.heads:
        q, k, v = ch.tm(Qc, h), ch.tm(Kc, h), ch.tm(ch.V, h)
        Osr, Lsr = O.sparse_attention_rows(q, k, v, masks[h], wl.block_q, wl.block_k, ch.scale,
                                           ch.rows)
        check_attention(ch.out_rows(out, h), Osr, f"{wl.name} {what} O h{h}")
        check_close(to64(lse)[h, ch.rows], Lsr, LSE_ABS, f"{wl.name} {what} LSE h{h}")


def release(ch):
    del ch.pipe, ch.Qd, ch.Kd, ch.Vd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wl", [workloads.WAN13B, workloads.WAN14B, workloads.HUNYUAN],
                         ids=lambda w: w.name)
def test_chain_full_size(wl):
    """Warm-up, tau calibrated to the workload's kept-block target, mask, and
    the workload's sparse calls (4 on perturbed Q/K for the Wan2.1-14B
    shape, reusing the warm-up's CSR; one on the warm-up's own Q/K
    otherwise)."""
    need_gpu()
    ch = Chain(wl)
    p = ch.pipe
    p.warmup_call(ch.Qd, ch.Kd, ch.Vd, None)
    tau = calibrate_tau(p, wl.kept_target)
    out, lse = ch.warmup(tau)
    kept = p.kept_fraction()
    assert abs(kept - wl.kept_target) < 0.02, kept
    check_warmup(ch, out, lse)
    masks = check_radius_and_mask(ch, wl.vote)
    if wl.sparse_calls > 1:
        for c in range(1, wl.sparse_calls + 1):
            Qc = inputs.perturb(ch.Q, wl.seed, c, 0)
            Kc = inputs.perturb(ch.K, wl.seed, c, 1)
            assert not torch.equal(Qc, ch.Q)
            o, l_ = ch.sparse(Qc.to(ch.dev), Kc.to(ch.dev))
            check_sparse(ch, masks, o, l_, Qc, Kc, f"sparse call {c}")
    else:
        o, l_ = ch.sparse(ch.Qd, ch.Kd)
        check_sparse(ch, masks, o, l_, ch.Q, ch.K, "sparse call")
    release(ch)


@pytest.mark.parametrize("grid,heads,d,block,vote,gamma,target", [
    ((5, 13, 22), 2, 64, 64, 1, 0.3, 0.6),     # N = 1430: 23 64-blocks, ragged tail of 22 tokens
    ((3, 18, 29), 3, 128, 128, 4, 0.5, 0.55),  # N = 1566: 13 128-blocks, ragged tail of 30 tokens
    ((3, 16, 43), 2, 128, 64, 16, 0.2, 0.35),  # N = 2064: 33 64-blocks (odd), last one 16 tokens
])
def test_chain_mid_size_every_element(grid, heads, d, block, vote, gamma, target):
    """The whole chain through the Pipeline at sizes the oracle covers in
    full: every element of the warm-up's O, H and LSE, every radius, the
    whole CSR bit for bit (given the GPU's fp32 radii) and every element of
    two sparse calls on perturbed Q/K over the warm-up's CSR."""
    need_gpu()
    wl = workloads.Workload(name=f"mid_{grid}", F=grid[0], H=grid[1], W=grid[2], heads=heads,
                            d=d, dtype="bf16", block_q=block, block_k=block, gamma=gamma,
                            vote=vote, seed=11, kept_target=target, sparse_calls=2)
    nnz, size = chain_every_element(wl)
    assert 0 < nnz < size


def chain_every_element(wl):
    """Runs the chain for `wl` (tau calibrated to wl.kept_target, or wl.tau)
    and compares every output with the oracle; returns (nnz, mask size)."""
    heads, d, block, vote, gamma = wl.heads, wl.d, wl.block_q, wl.vote, wl.gamma
    dev = torch.device("cuda", 0)
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, heads, d, wl.seed, wl.q_scale, "bf16")
    pipe = Pipeline(wl, dev)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    pipe.vote = vote
    if wl.kept_target is not None:
        pipe.warmup_call(Qd, Kd, Vd, None)
        pipe.tau = calibrate_tau(pipe, wl.kept_target)
    else:
        pipe.tau = wl.tau
    out = torch.empty_like(Qd)
    lse = torch.empty(heads, wl.N, dtype=torch.float32, device=dev)
    pipe.warmup_call(Qd, Kd, Vd, None, out=out, lse=lse)
    torch.cuda.synchronize()
    assert tra.tra_get_device_error() == 0
    pi = O.tile_major_order(*(wl.F, wl.H, wl.W), wl.tile)
    c = O.token_coords(wl.F, wl.H, wl.W)[pi]
    scale = 1.0 / math.sqrt(d)
    tm = lambda X: O.permute(to64(X), pi)  # noqa: E731
    Or, Hr, Lr = O.dense_attention_entropy(tm(Q), tm(K), tm(V), scale)
    check_attention(out, O.inverse_permute(Or, pi), "warm-up O")
    check_close(pipe.H, Hr, H_ABS, "H")
    check_close(lse, Lr, LSE_ABS, "LSE")
    tau32, gamma32 = float(np.float32(pipe.tau)), float(np.float32(gamma))
    rg, phig, Hg = pipe.r.cpu().numpy(), pipe.phi.cpu().numpy(), to64(pipe.H)
    for h in range(heads):
        assert np.allclose(rg[h], O.radius(Hg[h], c[:, 2], tau32, gamma32, wl.F, wl.N),
                           rtol=2e-6, atol=0)
    masks = np.stack([O.block_mask(rg[h], phig, c, block, block, vote) for h in range(heads)])
    rp_ref, ci_ref = O.to_csr(masks)
    nnz = int(pipe.nnz.item())
    assert nnz == len(ci_ref)
    assert np.array_equal(pipe.row_ptr.cpu().numpy(), rp_ref.ravel())
    assert np.array_equal(pipe.col_idx[:nnz].cpu().numpy(), ci_ref)
    for call in range(1, wl.sparse_calls + 1):
        Qc, Kc = inputs.perturb(Q, wl.seed, call, 0), inputs.perturb(K, wl.seed, call, 1)
        o = torch.empty_like(Qd)
        l_ = torch.empty_like(lse)
        pipe.sparse_call(Qc.to(dev), Kc.to(dev), Vd, None, out=o, lse=l_)
        torch.cuda.synchronize()
        assert tra.tra_get_device_error() == 0
        Osr, Lsr = O.sparse_attention(tm(Qc), tm(Kc), tm(V), masks, block, block, scale)
        check_attention(o, O.inverse_permute(Osr, pi), f"sparse call {call} O")
        check_close(l_, Lsr, LSE_ABS, f"sparse call {call} LSE")
    return nnz, masks.size


@pytest.fixture(scope="module")
def sweep_chain():
    need_gpu()
    ch = Chain(workloads.SWEEP)
    out, lse = ch.warmup(1.0)
    ch.warm = (out, lse)
    yield ch
    release(ch)


def test_sweep_warmup(sweep_chain):
    """The density sweep's own inputs (seed 4): dense warm-up O, H and LSE;
    its 100% point is this dense call."""
    check_warmup(sweep_chain, *sweep_chain.warm)


@pytest.mark.parametrize("vote", workloads.SWEEP.sweep_votes)
@pytest.mark.parametrize("target", [0.09, 0.40])
def test_sweep_points(sweep_chain, vote, target):
    """Sweep points: tau calibrated to the target at this vote threshold on
    the warm-up's entropy, then the mask and the block-sparse call."""
    ch = sweep_chain
    p = ch.pipe
    p.vote = vote
    tau = calibrate_tau(p, target)
    p.tau = tau
    p.mask(tau)
    torch.cuda.synchronize()
    assert abs(p.kept_fraction() - target) < 0.01, p.kept_fraction()
    masks = check_radius_and_mask(ch, vote)
    # the sweep times the block-sparse call on the warm-up's own inputs
    o, l_ = ch.sparse(ch.Qd, ch.Kd)
    check_sparse(ch, masks, o, l_, ch.Q, ch.K, f"sweep v{vote} {target:.0%}")
