"""Seeded synthetic inputs, shared by the CUDA path's tests/bench and the oracle.

This module holds no arithmetic of the method itself: it only draws random
numbers and shapes them into Q, K, V tensors (and into stand-in entropies,
radii and block masks for stage-wise tests).  Every draw comes from numpy's
Philox4x32-10 counter-based generator keyed by (seed, tensor, head), so a
value never depends on how many other values were drawn before it.

Q/K/V recipe (stands in for Wan2.1 / HunyuanVideo activations, which are not
available): for every head a random Fourier feature of the token's grid
position, P = sqrt(2/d) * cos(Wh @ [x, y, t] + bh) with Wh ~ N(0, 0.3^2) and
bh ~ U[0, 2*pi); keys k = P + 0.5*N(0,1); queries q = s * (P + 0.5*N(0,1)) with
a per-token scale s log-uniform in q_scale; values v ~ N(0,1).  Tokens are in
the original (t, y, x) row-major order.  Values are rounded once to the
workload's element type (bf16 or fp32).
"""
from concurrent.futures import ThreadPoolExecutor
import math
import os

import numpy as np
import torch

# tensor ids of the Philox key
_T_FEAT, _T_K, _T_QS, _T_Q, _T_V = 0, 1, 2, 3, 4
_T_PERTURB = 16
_T_ENTROPY, _T_RADIUS, _T_MASK = 64, 65, 66


def _rng(seed: int, tensor: int, head: int) -> np.random.Generator:
    key = np.array([np.uint64(seed), np.uint64((tensor << 32) | head)], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def grid_coords(F: int, H: int, W: int) -> np.ndarray:
    """[N, 3] float64 (x, y, t) of every token in original order (t*H + y)*W + x."""
    t, y, x = np.meshgrid(np.arange(F), np.arange(H), np.arange(W), indexing="ij")
    return np.stack([x.ravel(), y.ravel(), t.ravel()], axis=1).astype(np.float64)


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def make_qkv(F, H, W, heads, d, seed, q_scale=(0.5, 4.0), dtype="bf16",
             head_offset=0):
    """Q, K, V as CPU torch tensors [heads, N, d] of `dtype` (bf16 or f32).

    `head_offset` selects the global head index of the first head, so a
    shard of a larger problem draws the same values as the whole."""
    N = F * H * W
    coords = grid_coords(F, H, W)
    Q = torch.empty((heads, N, d), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    lo, hi = math.log(q_scale[0]), math.log(q_scale[1])

    def one(h):
        gh = h + head_offset
        g = _rng(seed, _T_FEAT, gh)
        Wh = g.normal(0.0, 0.3, size=(d, 3))
        bh = g.uniform(0.0, 2.0 * math.pi, size=d)
        P = math.sqrt(2.0 / d) * np.cos(coords @ Wh.T + bh)
        K[h] = _round(P + 0.5 * _rng(seed, _T_K, gh).standard_normal((N, d)), dtype)
        s = np.exp(_rng(seed, _T_QS, gh).uniform(lo, hi, size=N))
        Q[h] = _round(s[:, None] * (P + 0.5 * _rng(seed, _T_Q, gh).standard_normal((N, d))), dtype)
        V[h] = _round(_rng(seed, _T_V, gh).standard_normal((N, d)), dtype)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(one, range(heads)))
    return Q, K, V


def perturb(X: torch.Tensor, seed: int, call: int, which: int, sigma=0.05,
            head_offset=0) -> torch.Tensor:
    """X + sigma*N(0,1), re-rounded to X's dtype.  `call` numbers the sparse
    call (1, 2, ...) and `which` the tensor (0 = Q, 1 = K): each gets its own
    stream, as in the cross-step reuse setting (inputs drift slightly between
    denoising steps)."""
    heads, N, d = X.shape
    out = torch.empty_like(X)
    dtype = "bf16" if X.dtype == torch.bfloat16 else "f32"

    def one(h):
        g = _rng(seed, _T_PERTURB + 2 * call + which, h + head_offset)
        out[h] = _round(X[h].float().numpy().astype(np.float64)
                        + sigma * g.standard_normal((N, d)), dtype)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(one, range(heads)))
    return out


def synthetic_entropy(heads, N, seed, lo, hi) -> np.ndarray:
    """Stand-in per-query entropies, float32 [heads, N], uniform in [lo, hi]."""
    out = np.empty((heads, N), dtype=np.float32)
    for h in range(heads):
        out[h] = _rng(seed, _T_ENTROPY, h).uniform(lo, hi, size=N)
    return out


def synthetic_radius(heads, N, seed, lo, hi, special=True) -> np.ndarray:
    """Stand-in per-query radii, float32 [heads, N], log-uniform in [lo, hi].
    With `special`, a few entries are set to the edge values 0, +inf and NaN."""
    out = np.empty((heads, N), dtype=np.float32)
    for h in range(heads):
        g = _rng(seed, _T_RADIUS, h)
        out[h] = np.exp(g.uniform(math.log(lo), math.log(hi), size=N))
        if special and N >= 8:
            idx = g.choice(N, size=3, replace=False)
            out[h, idx[0]] = 0.0
            out[h, idx[1]] = np.inf
            out[h, idx[2]] = np.nan
    return out


def synthetic_block_mask(heads, nqb, nkb, seed, density, diagonal=True) -> np.ndarray:
    """Random kept-block pattern, bool [heads, nqb, nkb], each block kept with
    probability `density`; with `diagonal`, block (i, i * nkb // nqb) is kept."""
    out = np.empty((heads, nqb, nkb), dtype=bool)
    for h in range(heads):
        out[h] = _rng(seed, _T_MASK, h).random((nqb, nkb)) < density
        if diagonal:
            out[h, np.arange(nqb), (np.arange(nqb) * nkb) // nqb] = True
    return out


def csr_from_block_mask(mask: np.ndarray):
    """(row_ptr int32 [heads, nqb+1] of global offsets, col_idx int32 [nnz]):
    the kept key blocks of every (head, query block) row, ascending."""
    heads, nqb, nkb = mask.shape
    counts = mask.reshape(heads * nqb, nkb).sum(axis=1)
    starts = np.concatenate([[0], np.cumsum(counts)])
    row_ptr = np.empty((heads, nqb + 1), dtype=np.int64)
    for h in range(heads):
        row_ptr[h] = starts[h * nqb: h * nqb + nqb + 1]
    col_idx = np.nonzero(mask.reshape(heads * nqb, nkb))[1]
    return row_ptr.astype(np.int32), col_idx.astype(np.int32)
