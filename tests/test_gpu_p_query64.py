"""Block-sparse attention with 64-token query blocks at d = 128 (the
Wan2.1-1.3B shape's blocks): two query blocks share a 128-row tile and run the
ascending union of their CSR rows, each row leaving out the entries its own
block does not keep.  Parity with the fp64 oracle through the C ABI, at the
same tolerances as the other attention tests (output max abs 2e-2, mean abs
2e-3; LSE abs 1e-3), on the cases this path makes special: the running max
and its lazy rescale across super-blocks, keys that are not valid in the last
super-block (ragged tails, odd-length rows whose last super-block has one
64-key entry), empty rows, rows kept whole against the dense pass, the uniform
closed form, and the row checks that skip and report a malformed row."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra
from oracle import tra_oracle as O
from tests.gpu_util import LSE_ABS, check_attention, check_close, need_gpu, to64

pytestmark = pytest.mark.gpu

D = 128


def run(Q, K, V, row_ptr, col_idx, bq, bk, expect_code=0):
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    O_ = torch.full_like(Qd, 3.0)
    L = torch.full((Q.shape[0], Q.shape[1]), 3.0, dtype=torch.float32, device="cuda")
    rp = torch.as_tensor(np.asarray(row_ptr, np.int32).ravel()).cuda()
    ci = np.asarray(col_idx, np.int32)
    ci = torch.as_tensor(ci if ci.size else np.zeros(1, np.int32)).cuda()
    tra.tra_block_sparse_attn(Qd, Kd, Vd, O_, rp, ci, bq, bk, lse=L)
    torch.cuda.synchronize()
    code = tra.tra_get_device_error()
    assert code == expect_code
    return O_, L


def sparse_vs_oracle(Q, K, V, mask, bq, bk, what):
    row_ptr, col_idx = inputs.csr_from_block_mask(mask)
    O_, L = run(Q, K, V, row_ptr, col_idx, bq, bk)
    Or, Lr = O.sparse_attention(to64(Q), to64(K), to64(V), mask, bq, bk, 1.0 / math.sqrt(D))
    check_attention(O_, Or, what)
    check_close(L, Lr, LSE_ABS, "LSE " + what)
    return O_, L


@pytest.mark.parametrize("N,bk,density,seed", [
    (1000, 64, 0.3, 1),     # ragged query and key tails (1000 = 15 * 64 + 40)
    (1000, 128, 0.4, 2),    # 128-key blocks: one list entry per super-block
    (4096, 64, 0.15, 3),    # several tiles per head, odd and even row lengths
    (777, 64, 0.9, 4),      # dense rows, odd last super-blocks
    (130, 64, 0.5, 5),      # three query blocks, the last of 2 rows
])
def test_random_masks(N, bk, density, seed):
    need_gpu()
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(2, N, D, generator=g) * 2).to(torch.bfloat16)
    K = torch.randn(2, N, D, generator=g).to(torch.bfloat16)
    V = torch.randn(2, N, D, generator=g).to(torch.bfloat16)
    nqb, nkb = -(-N // 64), -(-N // bk)
    mask = inputs.synthetic_block_mask(2, nqb, nkb, seed=seed, density=density)
    mask[0, 0, :] = False                     # an empty row: O = 0, LSE = -inf
    O_, L = sparse_vs_oracle(Q, K, V, mask, 64, bk, f"N={N} bk={bk}")
    assert bool((O_[0, :64] == 0).all()) and bool(torch.isneginf(L[0, :64]).all())


@pytest.mark.parametrize("order", ["rising", "falling", "late_spike"])
def test_running_max_across_blocks(order):
    """The reference max moves only when a block exceeds it by more than
    2^8: scores that rise block after block rescale Z and O many times,
    falling scores never do, and a single key far above everything (a jump of
    about 200 in log2 units) in the last block rescales once by a factor that
    flushes all earlier terms to zero."""
    need_gpu()
    N = 2048
    g = torch.Generator().manual_seed(17)
    K = torch.randn(1, N, D, generator=g)
    Q = torch.randn(1, N, D, generator=g) * 2
    V = torch.randn(1, N, D, generator=g)
    if order == "rising":
        K *= torch.linspace(0.1, 6.0, N)[None, :, None]
    elif order == "falling":
        K *= torch.linspace(6.0, 0.1, N)[None, :, None]
    else:
        Q[0, :, 0] = 40.0
        K[0, N - 5, :] = 0.0
        K[0, N - 5, 0] = 40.0               # score ~141 (about 204 in log2 units) for key N - 5
    Qb, Kb, Vb = (t.to(torch.bfloat16) for t in (Q, K, V))
    nb = N // 64
    mask = np.ones((1, nb, nb), bool)
    sparse_vs_oracle(Qb, Kb, Vb, mask, 64, 64, order)
    half = inputs.synthetic_block_mask(1, nb, nb, seed=5, density=0.5)
    half[0, :, nb - 1] = True
    sparse_vs_oracle(Qb, Kb, Vb, half, 64, 64, order + " (half the blocks)")


def test_uniform_scores_average_the_kept_keys():
    """Q = 0: every kept key has weight 1 / (kept keys), so O is the mean of
    V over the row's kept tokens and LSE = ln(kept tokens), exactly the
    closed form (no oracle involved)."""
    need_gpu()
    N = 1000
    g = torch.Generator().manual_seed(23)
    V = torch.randn(1, N, D, generator=g).to(torch.bfloat16)
    K = torch.randn(1, N, D, generator=g).to(torch.bfloat16)
    Q = torch.zeros(1, N, D, dtype=torch.bfloat16)
    nb = -(-N // 64)
    rows = {q: sorted({q, (q * 7) % nb, nb - 1}) for q in range(nb)}
    rp, ci = [0], []
    for q in range(nb):
        ci += rows[q]
        rp.append(len(ci))
    O_, L = run(Q, K, V, rp, ci, 64, 64)
    v = to64(V)[0]
    lse = to64(L)[0]
    for q in range(nb):
        keys = np.concatenate([np.arange(kb * 64, min(N, kb * 64 + 64)) for kb in rows[q]])
        qs = slice(q * 64, min(N, q * 64 + 64))
        got = O_[0, qs]
        check_attention(got, np.broadcast_to(v[keys].mean(axis=0), tuple(got.shape)), f"mean V row {q}")
        assert np.allclose(lse[qs], math.log(keys.size), atol=LSE_ABS, rtol=0)


def test_all_blocks_kept_equals_dense():
    need_gpu()
    N = 1500
    g = torch.Generator().manual_seed(29)
    Q, K, V = ((torch.randn(2, N, D, generator=g) * s).to(torch.bfloat16) for s in (2, 1, 1))
    nb = -(-N // 64)
    Os, Ls = sparse_vs_oracle(Q, K, V, np.ones((2, nb, nb), bool), 64, 64, "all kept")
    Od = torch.empty_like(Os)
    H = torch.empty(2, N, dtype=torch.float32, device="cuda")
    Ld = torch.empty_like(H)
    tra.tra_dense_attn_entropy(Q.cuda(), K.cuda(), V.cuda(), Od, H, Ld)
    assert tra.tra_get_device_error() == 0
    check_attention(Os, to64(Od), "sparse (all kept) vs dense")
    check_close(Ls, to64(Ld), 1e-4, "LSE vs dense")


def test_malformed_and_invalid_rows_are_skipped_and_reported():
    """A row that is not strictly ascending within [0, nKB), or whose start
    is negative, or that holds more than nKB entries, is skipped (O = 0,
    LSE = -inf) and reported as an invalid CSR row (code 10); the other rows
    are exact."""
    need_gpu()
    N, B = 1024, 64
    nb = N // B
    rows = {q: [q] for q in range(nb)}
    rows.update({2: [5, 3, 7],                  # unsorted
                 5: [1, 1, 4],                  # a repeated entry
                 6: [3, nb + 83],               # an entry past nKB
                 9: [0, 2, 9],
                 11: list(range(nb)) + [0]})    # more than nKB entries
    bad = {2, 5, 6, 11}
    rp, ci = [0], []
    for q in range(nb):
        ci += rows[q]
        rp.append(len(ci))
    g = torch.Generator().manual_seed(31)
    Q, K, V = (torch.randn(1, N, D, generator=g).to(torch.bfloat16) for _ in range(3))
    O_, L = run(Q, K, V, rp, ci, B, B, expect_code=10)
    mask = np.zeros((1, nb, nb), bool)
    for q in range(nb):
        if q not in bad:
            mask[0, q, rows[q]] = True
    Or, Lr = O.sparse_attention(to64(Q), to64(K), to64(V), mask, B, B, 1.0 / math.sqrt(D))
    for q in bad:
        assert bool((O_[0, q * B:(q + 1) * B] == 0).all())
        assert bool(torch.isneginf(L[0, q * B:(q + 1) * B]).all())
    check_attention(O_, Or, "O with malformed rows")
    good = np.concatenate([np.arange(q * B, (q + 1) * B) for q in range(nb) if q not in bad])
    assert np.allclose(to64(L)[0, good], Lr[0, good], atol=1e-3, rtol=0)


def test_negative_row_start_is_skipped_and_reported():
    need_gpu()
    N, B = 512, 64
    nb = N // B
    rp = list(range(nb + 1))
    ci = list(range(nb))
    rp[0] = -3
    g = torch.Generator().manual_seed(37)
    Q, K, V = (torch.randn(1, N, D, generator=g).to(torch.bfloat16) for _ in range(3))
    O_, L = run(Q, K, V, rp, ci, B, B, expect_code=10)
    assert bool((O_[0, :B] == 0).all()) and bool(torch.isneginf(L[0, :B]).all())
    mask = np.zeros((1, nb, nb), bool)
    for q in range(1, nb):
        mask[0, q, q] = True
    Or, _ = O.sparse_attention(to64(Q), to64(K), to64(V), mask, B, B, 1.0 / math.sqrt(D))
    check_attention(O_[:, B:], Or[:, B:], "rows after the skipped one")
