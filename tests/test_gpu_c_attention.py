"""GPU parity of the tcgen05 attention kernels (dense + entropy, block-sparse)
against the fp64 oracle, through the C ABI.  Tolerances: output max abs
2e-2 and mean abs 2e-3; entropy and LSE abs 1e-3."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import (H_ABS, LSE_ABS, check_attention, check_close, need_gpu, to64)

pytestmark = pytest.mark.gpu


def gpu_dense(Q, K, V, with_lse=True):
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    heads, N, d = Q.shape
    O_ = torch.empty_like(Qd)
    H = torch.empty(heads, N, dtype=torch.float32, device="cuda")
    L = torch.empty_like(H) if with_lse else None
    tra.tra_dense_attn_entropy(Qd, Kd, Vd, O_, H, L)
    assert tra.tra_get_device_error() == 0
    return O_, H, L


def gpu_sparse(Q, K, V, mask, bq, bk):
    row_ptr, col_idx = inputs.csr_from_block_mask(mask)
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    O_ = torch.empty_like(Qd)
    L = torch.empty(Q.shape[0], Q.shape[1], dtype=torch.float32, device="cuda")
    rp = torch.from_numpy(row_ptr.ravel()).cuda()
    ci = torch.from_numpy(col_idx if col_idx.size else np.zeros(1, np.int32)).cuda()
    tra.tra_block_sparse_attn(Qd, Kd, Vd, O_, rp, ci, bq, bk, lse=L)
    assert tra.tra_get_device_error() == 0
    return O_, L


def rand_qkv(heads, N, d, seed, qscale=1.0):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(heads, N, d, generator=g) * qscale).to(torch.bfloat16)
    K = torch.randn(heads, N, d, generator=g).to(torch.bfloat16)
    V = torch.randn(heads, N, d, generator=g).to(torch.bfloat16)
    return Q, K, V


# ------------------------------------------------------------------ dense

@pytest.mark.parametrize("heads,N,d", [(1, 128, 64), (1, 128, 128), (2, 256, 64), (2, 1000, 128),
                                       (1, 60, 64), (1, 1, 128), (3, 777, 64), (1, 2560, 128)])
def test_dense_entropy_random(heads, N, d):
    need_gpu()
    Q, K, V = rand_qkv(heads, N, d, seed=N + d, qscale=2.0)
    O_, H, L = gpu_dense(Q, K, V)
    Or, Hr, Lr = O.dense_attention_entropy(to64(Q), to64(K), to64(V), 1.0 / math.sqrt(d))
    check_attention(O_, Or, "O")
    check_close(H, Hr, H_ABS, "H")
    check_close(L, Lr, LSE_ABS, "LSE")


def test_dense_tiny_workload():
    """Tiny workload: fp32 inputs cast to bf16 by the permute, then dense."""
    need_gpu()
    w = workloads.TINY
    Q, K, V = inputs.make_qkv(w.F, w.H, w.W, w.heads, w.d, w.seed, w.q_scale, "f32")
    grid = (w.F, w.H, w.W)
    tm = []
    for X in (Q, K, V):
        Y = torch.empty(X.shape, dtype=torch.bfloat16, device="cuda")
        tra.tra_tile_major_permute(X.cuda(), Y, grid, w.tile)
        tm.append(Y.cpu())
    O_, H, L = gpu_dense(*tm)
    pi = O.tile_major_order(*grid, w.tile)
    # the oracle is fed the same bf16-rounded values (rounding done by torch here)
    ref_in = [O.permute(to64(X.to(torch.bfloat16)), pi) for X in (Q, K, V)]
    Or, Hr, Lr = O.dense_attention_entropy(*ref_in, 1.0 / math.sqrt(w.d))
    check_attention(O_, Or, "O")
    check_close(H, Hr, H_ABS, "H")
    check_close(L, Lr, LSE_ABS, "LSE")


def test_dense_uniform_scores_entropy_is_log_n():
    need_gpu()
    for N, d in ((300, 64), (5000, 128)):
        _, K, V = rand_qkv(2, N, d, seed=1)
        Q = torch.zeros(2, N, d, dtype=torch.bfloat16)
        O_, H, L = gpu_dense(Q, K, V)
        check_close(H, np.full((2, N), math.log(N)), H_ABS, "H uniform")
        check_close(L, np.full((2, N), math.log(N)), LSE_ABS, "LSE uniform")
        # output is the mean of V
        check_attention(O_, np.broadcast_to(to64(V).mean(axis=1, keepdims=True), (2, N, d)), "mean V")


def test_dense_one_hot_entropy_is_zero():
    need_gpu()
    N, d = 700, 64
    Q = torch.zeros(1, N, d)
    K = torch.zeros(1, N, d)
    V = torch.randn(1, N, d, generator=torch.Generator().manual_seed(3))
    Q[0, :, 0] = 400.0      # scaled score 50 against key 123, 0 against the rest
    K[0, 123, 0] = 1.0
    Qb, Kb, Vb = (t.to(torch.bfloat16) for t in (Q, K, V))
    O_, H, _ = gpu_dense(Qb, Kb, Vb)
    check_close(H, np.zeros((1, N)), H_ABS, "H one-hot")
    check_attention(O_, np.broadcast_to(to64(Vb)[:, 123:124], (1, N, d)), "O one-hot")


def test_dense_large_score_range_rescales():
    """Rows whose running maximum grows block after block exercise the lazy
    rescale of the output accumulator."""
    need_gpu()
    heads, N, d = 1, 1024, 128
    g = torch.Generator().manual_seed(9)
    K = torch.randn(heads, N, d, generator=g)
    K *= torch.linspace(0.1, 6.0, N)[None, :, None]       # later keys score higher
    Q = torch.randn(heads, N, d, generator=g) * 2
    V = torch.randn(heads, N, d, generator=g)
    Q, K, V = (t.to(torch.bfloat16) for t in (Q, K, V))
    O_, H, L = gpu_dense(Q, K, V)
    Or, Hr, Lr = O.dense_attention_entropy(to64(Q), to64(K), to64(V), 1.0 / math.sqrt(d))
    check_attention(O_, Or, "O")
    check_close(H, Hr, H_ABS, "H")
    check_close(L, Lr, LSE_ABS, "LSE")


# ------------------------------------------------------------------ sparse

SPARSE = [  # heads, N, d, bq, bk, density
    (2, 1000, 128, 128, 128, 0.3), (2, 1000, 128, 64, 64, 0.3), (2, 256, 64, 16, 16, 0.3),
    (2, 1000, 64, 128, 64, 0.25), (2, 1000, 128, 64, 128, 0.4), (2, 600, 128, 16, 64, 0.3),
    (1, 3000, 128, 128, 128, 0.1), (1, 700, 64, 16, 128, 0.5), (2, 333, 128, 128, 16, 0.2),
    # two 64-row query blocks per tile at d = 64; an odd query-block count,
    # whose last tile holds one block (its CSR row read directly)
    (2, 1000, 64, 64, 64, 0.3), (1, 777, 64, 64, 128, 0.35), (2, 1050, 128, 64, 64, 0.3),
]


@pytest.mark.parametrize("heads,N,d,bq,bk,density", SPARSE)
def test_sparse_random_mask(heads, N, d, bq, bk, density):
    need_gpu()
    Q, K, V = rand_qkv(heads, N, d, seed=N * bq + bk, qscale=2.0)
    nqb, nkb = -(-N // bq), -(-N // bk)
    mask = inputs.synthetic_block_mask(heads, nqb, nkb, seed=N + bk, density=density)
    O_, L = gpu_sparse(Q, K, V, mask, bq, bk)
    Or, Lr = O.sparse_attention(to64(Q), to64(K), to64(V), mask, bq, bk, 1.0 / math.sqrt(d))
    check_attention(O_, Or, "O")
    check_close(L, Lr, LSE_ABS, "LSE")


def test_sparse_all_ones_equals_dense_and_empty_rows():
    need_gpu()
    heads, N, d = 2, 900, 128
    Q, K, V = rand_qkv(heads, N, d, seed=77)
    nb = -(-N // 128)
    full = np.ones((heads, nb, nb), bool)
    Os, Ls = gpu_sparse(Q, K, V, full, 128, 128)
    Od, _, Ld = gpu_dense(Q, K, V)
    check_attention(Os, to64(Od), "sparse(all) vs dense")
    check_close(Ls, to64(Ld), 1e-4, "LSE")
    empty = full.copy()
    empty[0, 2, :] = False
    empty[1, nb - 1, :] = False
    Oe, Le = gpu_sparse(Q, K, V, empty, 128, 128)
    oe = to64(Oe)
    assert np.all(oe[0, 256:384] == 0) and np.all(oe[1, (nb - 1) * 128:] == 0)
    le = to64(Le)
    assert np.all(le[0, 256:384] == -np.inf) and np.all(le[1, (nb - 1) * 128:] == -np.inf)
    # union mode (64-row query blocks): one block row empty, its partner not
    nq64, nk64 = -(-N // 64), -(-N // 64)
    m64 = inputs.synthetic_block_mask(heads, nq64, nk64, seed=1, density=0.3)
    m64[0, 3, :] = False
    O6, L6 = gpu_sparse(Q, K, V, m64, 64, 64)
    Or, Lr = O.sparse_attention(to64(Q), to64(K), to64(V), m64, 64, 64, 1.0 / math.sqrt(d))
    check_attention(O6, Or, "union")
    check_close(L6, Lr, LSE_ABS, "LSE union")


# ---------------------------------------------------------------- full size

FULL = [workloads.WAN13B, workloads.WAN14B, workloads.HUNYUAN]


@pytest.mark.parametrize("wl", FULL, ids=lambda w: w.name)
def test_full_size_dense_and_sparse_sampled(wl):
    """Full-size launches (all heads, as the bench runs them); the oracle
    checks sampled query rows: the first, a middle and the last (partial)
    query tile of a few heads."""
    need_gpu()
    Q, K, V = inputs.make_qkv(wl.F, wl.H, wl.W, wl.heads, wl.d, wl.seed, wl.q_scale, "bf16")
    O_, H, L = gpu_dense(Q, K, V)
    N, d = wl.N, wl.d
    bq, bk = wl.block_q, wl.block_k
    nqb, nkb = -(-N // bq), -(-N // bk)
    mask = inputs.synthetic_block_mask(wl.heads, nqb, nkb, seed=wl.seed, density=0.12)
    Os, Ls = gpu_sparse(Q, K, V, mask, bq, bk)
    rng = np.random.default_rng(wl.seed)
    heads = sorted({0, wl.heads - 1, int(rng.integers(wl.heads))})
    last = (N - 1) // 128 * 128
    rows = np.unique(np.concatenate([np.arange(0, 128), np.arange(N // 2 - 64, N // 2 + 64),
                                     np.arange(last, N), rng.integers(0, N, 64)]))
    Hn, Ln, Lsn = to64(H), to64(L), to64(Ls)
    scale = 1.0 / math.sqrt(d)
    for h in heads:
        q, k, v = to64(Q[h]), to64(K[h]), to64(V[h])
        Or, Hr, Lr = O.attention_rows(q, k, v, scale, rows)
        check_attention(O_[h][rows], Or, f"dense O h{h}")
        check_close(Hn[h, rows], Hr, H_ABS, f"H h{h}")
        check_close(Ln[h, rows], Lr, LSE_ABS, f"LSE h{h}")
        Osr, Lsr = O.sparse_attention_rows(q, k, v, mask[h], bq, bk, scale, rows)
        check_attention(Os[h][rows], Osr, f"sparse O h{h}")
        check_close(Lsn[h, rows], Lsr, LSE_ABS, f"sparse LSE h{h}")
    assert bool(torch.isfinite(O_).all()) and bool(torch.isfinite(Os).all())
    assert np.isfinite(Hn).all()
    assert (Hn <= math.log(N) + H_ABS).all() and (Hn >= -H_ABS).all()


@pytest.mark.parametrize("d", [64, 128])
def test_union_list_and_walk_fallback_at_the_cap(d):
    """At d = 64, 64-row query blocks pair up in 128-row tiles whose
    key-block list is the merged union of two CSR rows: held in shared memory
    up to 384 entries, walked from the two rows beyond.  Tiles are planted at
    exactly 384 and 385 entries, and with interleaved rows (mixed membership
    bits) on both sides of the cap; every other row keeps its diagonal block.
    The same at both head dimensions."""
    need_gpu()
    N, B = 32768, 64
    nb = N // B
    mask = np.zeros((1, nb, nb), bool)
    mask[0, np.arange(nb), np.arange(nb)] = True
    plants = {
        2: np.arange(0, 300), 3: np.arange(200, 384),            # union 384: list
        6: np.arange(0, 300), 7: np.arange(200, 385),            # union 385: walk
        10: np.arange(0, nb, 2), 11: np.arange(1, nb, 2),        # union 512, disjoint: walk
        14: np.arange(0, 300, 2), 15: np.arange(0, 300, 3),      # union 200, shared entries: list
    }
    for q, cols in plants.items():
        mask[0, q] = False
        mask[0, q, cols] = True
    unions = {q: len(set(plants[q]) | set(plants[q + 1])) for q in (2, 6, 10, 14)}
    assert unions == {2: 384, 6: 385, 10: 512, 14: 200}
    Q, K, V = rand_qkv(1, N, d, seed=384, qscale=2.0)
    Os, Ls = gpu_sparse(Q, K, V, mask, B, B)
    rows = np.concatenate([np.arange(q * B, (q + 1) * B) for q in plants] +
                          [np.arange(0, 64), np.arange(N - 64, N)])
    q, k, v = to64(Q[0]), to64(K[0]), to64(V[0])
    Osr, Lsr = O.sparse_attention_rows(q, k, v, mask[0], B, B, 1.0 / math.sqrt(d), rows)
    check_attention(Os[0][rows], Osr, "sparse O at the union cap")
    check_close(to64(Ls)[0, rows], Lsr, LSE_ABS, "sparse LSE at the union cap")


@pytest.mark.parametrize("scale", [0.03, 0.4])
def test_dense_and_sparse_with_a_given_scale(scale):
    """The softmax scale is an argument of both calls (the default is
    1/sqrt(d)); a small scale flattens the rows, a large one sharpens them."""
    need_gpu()
    heads, N, d, B = 2, 700, 128, 64
    Q, K, V = rand_qkv(heads, N, d, seed=int(scale * 1000))
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    O_ = torch.empty_like(Qd)
    H = torch.empty(heads, N, dtype=torch.float32, device="cuda")
    L = torch.empty_like(H)
    tra.tra_dense_attn_entropy(Qd, Kd, Vd, O_, H, L, scale=scale)
    assert tra.tra_get_device_error() == 0
    Or, Hr, Lr = O.dense_attention_entropy(to64(Q), to64(K), to64(V), scale)
    check_attention(O_, Or, f"dense O scale {scale}")
    check_close(H, Hr, H_ABS, f"H scale {scale}")
    check_close(L, Lr, LSE_ABS, f"LSE scale {scale}")
    nb = -(-N // B)
    mask = inputs.synthetic_block_mask(heads, nb, nb, seed=7, density=0.3)
    rp, ci = inputs.csr_from_block_mask(mask)
    Os = torch.empty_like(Qd)
    Ls = torch.empty_like(H)
    tra.tra_block_sparse_attn(Qd, Kd, Vd, Os, torch.from_numpy(rp.ravel()).cuda(),
                              torch.from_numpy(ci).cuda(), B, B, lse=Ls, scale=scale)
    assert tra.tra_get_device_error() == 0
    Osr, Lsr = O.sparse_attention(to64(Q), to64(K), to64(V), mask, B, B, scale)
    check_attention(Os, Osr, f"sparse O scale {scale}")
    check_close(Ls, Lsr, LSE_ABS, f"sparse LSE scale {scale}")
