"""The chained Token Radius Attention calls of one attention layer, as the
benchmark runs them and the chained parity tests check them (Token Radius
Attention summary, §2 "TRA pipeline": dense warm-up attention with entropy,
entropy -> budget -> radius, the fused radius mask -> block-sparse CSR, and
block-sparse attention over the kept blocks, reused by later calls).

`Pipeline` owns the device buffers of one layer and issues every step through
the C ABI (`tra`): a warm-up call (tile-major permute of Q, K, V; dense
attention + entropy; radius; mask; inverse permute of O) and sparse calls
(permute; block-sparse attention over the warm-up's CSR; inverse permute).
`calibrate_tau` bisects tau on the kept-block fraction of the GPU mask.  This
module sequences calls and counts work; every step of the method runs in the
CUDA kernels.
"""
import math

import numpy as np
import torch

from . import tra


def kept_pair_tokens(row_ptr, col_idx, heads, N, bq, bk):
    """sum over kept (qb, kb) of |qb| * |kb| (tail blocks shorter), all heads."""
    nqb, nkb = -(-N // bq), -(-N // bk)
    rp = row_ptr.reshape(heads, nqb + 1)
    qsz = np.minimum(bq, N - np.arange(nqb) * bq).astype(np.int64)
    ksz = np.minimum(bk, N - np.arange(nkb) * bk).astype(np.int64)
    total = 0
    for h in range(heads):
        s, e = int(rp[h, 0]), int(rp[h, nqb])
        cols = col_idx[s:e]
        counts = np.diff(rp[h])
        rows = np.repeat(np.arange(nqb), counts)
        total += int((qsz[rows] * ksz[cols]).sum())
    return total


def full_csr(heads, N, block, device):
    """CSR that keeps every (query block, key block) pair."""
    nqb = nkb = -(-N // block)
    idx = torch.arange(heads * (nqb + 1), dtype=torch.int64)
    rp = (idx // (nqb + 1) * nqb + idx % (nqb + 1)) * nkb
    ci = torch.arange(nkb, dtype=torch.int32).repeat(heads * nqb)
    return rp.to(torch.int32).to(device), ci.to(device)


class Pipeline:
    """Device buffers and launches of one TRA layer (all calls through the C ABI)."""

    def __init__(self, wl, device):
        self.tra = tra
        self.wl = wl
        self.grid = (wl.F, wl.H, wl.W)
        h, N, d = wl.heads, wl.N, wl.d
        bf = dict(dtype=torch.bfloat16, device=device)
        self.Qtm, self.Ktm, self.Vtm = (torch.empty(h, N, d, **bf) for _ in range(3))
        self.Otm = torch.empty(h, N, d, **bf)
        self.O = torch.empty(h, N, d, **bf)
        self.H = torch.empty(h, N, dtype=torch.float32, device=device)
        self.r = torch.empty_like(self.H)
        self.phi = torch.empty(wl.F, dtype=torch.float32, device=device)
        self.nqb, self.nkb = wl.nqb, wl.nkb
        self.row_ptr = torch.empty(h * (self.nqb + 1), dtype=torch.int32, device=device)
        self.col_idx = torch.empty(h * self.nqb * self.nkb, dtype=torch.int32, device=device)
        self.nnz = torch.empty(1, dtype=torch.int32, device=device)
        self.ws = tra.workspace_tensor(
            tra.tra_mask_workspace_size(h, self.grid, wl.block_q, wl.block_k, wl.tile), device)
        self.launches = 0
        self.tau = 1.0
        self.vote = wl.vote

    # mask source: ("entropy" | "shared" | "radial", "disk" | "line"); the
    # parameter of mask() is tau for the entropy budgets and r0 for radial
    variant = ("entropy", "disk")

    def radius(self, param):
        w, t = self.wl, self.tra
        source, metric = self.variant
        if source == "radial":
            t.tra_radial_radius(self.r, self.grid, param, metric, w.tile, phi_out=self.phi)
        else:
            t.tra_budget_radius_ex(self.H, self.r, self.grid, param, w.gamma, source, metric,
                                   w.tile, phi_out=self.phi)

    def mask(self, param):
        w, t = self.wl, self.tra
        self.radius(param)
        t.tra_build_block_mask_ex(self.r, self.phi, self.grid, w.block_q, w.block_k, self.vote,
                                  self.row_ptr, self.col_idx, self.nnz, self.ws, self.variant[1],
                                  w.tile)
        self.launches += 5

    def _operands(self, Q, K, V, out, resident):
        """Kernel operands: the tile-major buffers, filled by permuting Q, K, V,
        or (resident) Q, K, V and out themselves, already in tile-major order."""
        if resident:
            return Q, K, V, out, 0
        for X, Y in ((Q, self.Qtm), (K, self.Ktm), (V, self.Vtm)):
            self.tra.tra_tile_major_permute(X, Y, self.grid, self.wl.tile)
        return self.Qtm, self.Ktm, self.Vtm, self.Otm, 4

    def warmup_call(self, Q, K, V, rec, out=None, resident=False, lse=None):
        """Dense warm-up call; `lse` ([heads, N] fp32, tile-major) optionally
        receives the log-sum-exp of every query."""
        t = self.tra
        out = self.O if out is None else out
        e = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        e[0].record()
        q, k, v, o, nperm = self._operands(Q, K, V, out, resident)
        e[1].record()
        t.tra_dense_attn_entropy(q, k, v, o, self.H, lse)
        e[2].record()
        t.tra_budget_radius(self.H, self.r, self.grid, self.tau, self.wl.gamma, self.wl.tile,
                            phi_out=self.phi)
        e[3].record()
        t.tra_build_block_mask(self.r, self.phi, self.grid, self.wl.block_q, self.wl.block_k,
                               self.vote, self.row_ptr, self.col_idx, self.nnz, self.ws,
                               self.wl.tile)
        e[4].record()
        if not resident:
            t.tra_inverse_permute(self.Otm, out, self.grid, self.wl.tile)
        e[5].record()
        self.launches += nperm + 1 + 1 + 4
        if rec is not None:
            rec.append(("warmup", e))

    def sparse_call(self, Q, K, V, rec, out=None, resident=False, lse=None):
        """Block-sparse call over the current CSR; `lse` as for warmup_call."""
        t = self.tra
        out = self.O if out is None else out
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        q, k, v, o, nperm = self._operands(Q, K, V, out, resident)
        e[1].record()
        t.tra_block_sparse_attn(q, k, v, o, self.row_ptr, self.col_idx, self.wl.block_q,
                                self.wl.block_k, lse=lse)
        e[2].record()
        if not resident:
            t.tra_inverse_permute(self.Otm, out, self.grid, self.wl.tile)
        e[3].record()
        self.launches += nperm + 1
        if rec is not None:
            rec.append(("sparse", e))

    def kept_fraction(self):
        return int(self.nnz.item()) / (self.wl.heads * self.nqb * self.nkb)


def calibrate_tau(pipe, target, log=None):
    """Bisection of log(tau) on the kept-block fraction (monotone in tau)."""
    lo, hi = math.log(1e-6), math.log(1e4)
    best = None
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        pipe.mask(math.exp(mid))
        f = pipe.kept_fraction()
        if best is None or abs(f - target) < abs(best[1] - target):
            best = (math.exp(mid), f)
        if abs(f - target) < 0.002:
            break
        if f > target:
            hi = mid
        else:
            lo = mid
    if log is not None:
        log(f"tau calibrated: tau={best[0]:.5g} kept={best[1]:.4f} (target {target})")
    return best[0]
