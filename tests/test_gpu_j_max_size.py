"""The largest problem the calls accept: N = 2^24 tokens (64 x 512 x 512),
d = 128, one head.  One tensor then holds 2^31 elements, so every offset
past 2^31 must be formed in 64-bit arithmetic.  The inputs are drawn on the
device; the oracle checks sampled rows: the tile-major permutation
(forward and inverse) against its own order, and block-sparse attention over
the diagonal blocks against exact attention within each sampled block."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import tra
from oracle import tra_oracle as O
from tests.gpu_util import check_attention, check_close, LSE_ABS, need_gpu, to64

pytestmark = pytest.mark.gpu

GRID = (64, 512, 512)
TILE = (1, 4, 4)
N = GRID[0] * GRID[1] * GRID[2]
D = 128


def device_randn(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


def sample_positions(rng):
    return np.unique(np.concatenate([np.arange(0, 64), np.arange(N - 64, N),
                                     np.arange(N // 2 - 32, N // 2 + 32), rng.integers(0, N, 256)]))


def test_permute_at_the_largest_size():
    need_gpu()
    assert N == 1 << 24
    X = device_randn((1, N, D), 1)
    Y = torch.empty_like(X)
    tra.tra_tile_major_permute(X, Y, GRID, TILE)
    pi = O.tile_major_order(*GRID, TILE)
    p = sample_positions(np.random.default_rng(1))
    idx = torch.from_numpy(pi[p]).cuda()
    assert torch.equal(Y[0, torch.from_numpy(p).cuda()], X[0, idx])
    Z = torch.empty_like(X)
    tra.tra_inverse_permute(Y, Z, GRID, TILE)
    rows = torch.from_numpy(sample_positions(np.random.default_rng(2))).cuda()
    assert torch.equal(Z[0, rows], X[0, rows])
    assert tra.tra_get_device_error() == 0


def test_block_sparse_attention_at_the_largest_size():
    need_gpu()
    B = 128
    nqb = N // B
    Q, K, V = device_randn((1, N, D), 2), device_randn((1, N, D), 3), device_randn((1, N, D), 4)
    O_ = torch.empty_like(Q)
    L = torch.empty(1, N, dtype=torch.float32, device="cuda")
    rp = torch.arange(nqb + 1, dtype=torch.int32, device="cuda")
    ci = torch.arange(nqb, dtype=torch.int32, device="cuda")
    tra.tra_block_sparse_attn(Q, K, V, O_, rp, ci, B, B, lse=L)
    assert tra.tra_get_device_error() == 0
    scale = 1.0 / math.sqrt(D)
    rng = np.random.default_rng(5)
    for qb in sorted({0, 1, nqb // 2, nqb - 1, *rng.integers(0, nqb, 4).tolist()}):
        sl = slice(qb * B, (qb + 1) * B)
        q, k, v = to64(Q[0, sl]), to64(K[0, sl]), to64(V[0, sl])
        Or, Lr, _ = O.softmax_attention(q, k, v, scale)
        check_attention(O_[0, sl], Or, f"O block {qb}")
        check_close(L[0, sl], Lr, LSE_ABS, f"LSE block {qb}")
