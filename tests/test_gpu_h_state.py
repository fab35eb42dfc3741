"""Failure detection and resumable state on the GPU.

The bounded-wait self-test waits on a barrier nothing completes: the wait
must give up after its limit, report TRA_ERR_TIMEOUT with its code, clear on
reading, and leave the context usable.  A layer's reuse state (entropy,
radii, mask, step index) saved after the warm-up and loaded into a fresh
layer must reproduce the original layer's next steps bit for bit."""
import io
import math
import time

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra
from entropy_adaptive_radius_b200.layer import ReusePolicy, TraLayer
from oracle import tra_oracle as O
from tests.gpu_util import check_attention, need_gpu, to64

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_and_context_survives():
    need_gpu()
    assert tra.tra_get_device_error() == 0
    flag = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    tra.tra_selftest_wait_timeout(50, flag)
    code = tra.tra_get_device_error()        # synchronises the stream
    dt = time.time() - t0
    assert code == 11
    assert int(flag[0].item()) == 0          # the wait gave up, it did not complete
    assert 0.045 < dt < 2.0
    assert tra.tra_get_device_error() == 0   # the word is cleared by reading it
    # the context still runs the attention kernels correctly
    g = torch.Generator().manual_seed(4)
    Q, K, V = (torch.randn(1, 300, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    O_ = torch.empty(1, 300, 64, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(1, 300, dtype=torch.float32, device="cuda")
    tra.tra_dense_attn_entropy(Q.cuda(), K.cuda(), V.cuda(), O_, H)
    assert tra.tra_get_device_error() == 0
    Or, _, _ = O.dense_attention_entropy(to64(Q), to64(K), to64(V), 1.0 / math.sqrt(64))
    check_attention(O_, Or, "O after the timeout")


def test_layer_state_round_trip_resumes_bit_for_bit():
    need_gpu()
    grid, heads, d = (4, 12, 16), 2, 64
    N = 4 * 12 * 16
    policy = ReusePolicy(warmup=1, refresh_every=3, refresh="entropy")
    kw = dict(tau=0.2, gamma=0.3, block_q=64, block_k=64, policy=policy)
    Q, K, V = inputs.make_qkv(*grid, heads, d, 7, (0.5, 4.0), "bf16")
    steps = [(inputs.perturb(Q, 7, c, 0), inputs.perturb(K, 7, c, 1), V) for c in range(1, 6)]
    a = TraLayer(grid, heads, d, **kw)
    a(Q.cuda(), K.cuda(), V.cuda())                      # warm-up: entropy and mask
    buf = io.BytesIO()
    torch.save(a.state_dict(), buf)
    buf.seek(0)
    b = TraLayer(grid, heads, d, **kw)
    b.load_state_dict(torch.load(buf))
    assert b.step_index == a.step_index == 1
    for q, k, v in steps:                                 # sparse steps and a refresh
        Oa = a(q.cuda(), k.cuda(), v.cuda())
        Ob = b(q.cuda(), k.cuda(), v.cuda())
        assert torch.equal(Oa, Ob)
        assert torch.equal(a.row_ptr, b.row_ptr)
    assert tra.tra_get_device_error() == 0
    c = TraLayer(grid, heads, d, tau=0.3, gamma=0.3, block_q=64, block_k=64, policy=policy)
    with pytest.raises(ValueError):
        c.load_state_dict(a.state_dict())


def bad_csr_case(N, B, bad_row, kind):
    """A CSR over nqb x nkb blocks whose row `bad_row` is invalid (longer
    than nkb, or with a negative start) and every other row keeps one key
    block.  Returns (row_ptr, col_idx, mask of what a valid call computes)."""
    nb = -(-N // B)
    rows = [[(q + 1) % nb] for q in range(nb)]
    rp, ci = [0], []
    for q in range(nb):
        if q == bad_row and kind == "long":
            ci += list(range(nb)) + [0]              # nkb + 1 entries
        else:
            ci += rows[q]
        rp.append(len(ci))
    rp = np.array(rp, np.int32)
    if kind == "negative":
        rp[bad_row] = -3                             # start of the bad row
    mask = np.zeros((1, nb, nb), bool)
    for q in range(nb):
        if q != bad_row:
            mask[0, q, rows[q][0]] = True
    return rp, np.array(ci, np.int32), mask


@pytest.mark.parametrize("B", [128, 64, 16])
@pytest.mark.parametrize("kind", ["long", "negative"])
def test_invalid_csr_row_is_skipped_and_reported(B, kind):
    need_gpu()
    N, d = 256, 64
    g = torch.Generator().manual_seed(B)
    Q, K, V = (torch.randn(1, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    # a negative start of row q also ends row q - 1 below its start, so the
    # negative case uses row 0; the long case a middle row
    bad = 0 if kind == "negative" else 1
    rp, ci, mask = bad_csr_case(N, B, bad, kind)
    O_ = torch.full((1, N, d), 7.0, dtype=torch.bfloat16, device="cuda")
    L = torch.empty(1, N, device="cuda")
    assert tra.tra_get_device_error() == 0
    tra.tra_block_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), O_, torch.from_numpy(rp).cuda(),
                              torch.from_numpy(ci).cuda(), B, B, lse=L)
    code = _c_code()
    assert code == (10, 8)                           # invalid CSR row, TRA_ERR_BAD_INPUT
    Or, Lr = O.sparse_attention(to64(Q), to64(K), to64(V), mask, B, B, 1.0 / math.sqrt(d))
    rows = slice(bad * B, (bad + 1) * B)
    assert bool((O_[0, rows] == 0).all())
    assert bool(torch.isneginf(L[0, rows]).all())
    check_attention(O_, Or, f"O with an invalid row ({kind}, B={B})")
    keep = np.isfinite(Lr[0])
    assert np.allclose(to64(L)[0, keep], Lr[0, keep], atol=1e-3, rtol=0)


def _c_code():
    """(device code, status) read through the C call itself."""
    import ctypes
    code = ctypes.c_int(0)
    s = tra.lib().tra_get_device_error(ctypes.byref(code), tra._stream(None))
    return code.value, s


def test_malformed_rows_of_a_two_block_tile_are_skipped():
    """With 64-row query blocks two CSR rows share a tile and its merged key
    list.  A row that is not strictly ascending within [0, nKB) (unsorted, a
    repeated entry, an entry out of range) is skipped and reported, and the
    other row of its tile is still computed exactly: a skipped row A leaves row
    B on the merged list, a skipped row B leaves row A on the one-row path."""
    need_gpu()
    N, d, B = 1024, 64, 64
    nb = N // B
    rows = {q: [q] for q in range(nb)}
    rows.update({2: [5, 3, 7], 3: [2, 3, 4],      # A unsorted, B kept
                 4: [0, 4, 9], 5: [1, 1, 4],      # B repeats an entry, A kept
                 6: [3, nb + 83], 7: [9, 8]})     # both malformed
    bad = {2, 5, 6, 7}
    rp, ci = [0], []
    for q in range(nb):
        ci += rows[q]
        rp.append(len(ci))
    mask = np.zeros((1, nb, nb), bool)
    for q in range(nb):
        if q not in bad:
            mask[0, q, rows[q]] = True
    g = torch.Generator().manual_seed(11)
    Q, K, V = (torch.randn(1, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    O_ = torch.full((1, N, d), 5.0, dtype=torch.bfloat16, device="cuda")
    L = torch.empty(1, N, device="cuda")
    assert tra.tra_get_device_error() == 0
    tra.tra_block_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), O_, torch.tensor(rp, dtype=torch.int32).cuda(),
                              torch.tensor(ci, dtype=torch.int32).cuda(), B, B, lse=L)
    assert _c_code() == (10, 8)
    Or, Lr = O.sparse_attention(to64(Q), to64(K), to64(V), mask, B, B, 1.0 / math.sqrt(d))
    for q in bad:
        assert bool((O_[0, q * B:(q + 1) * B] == 0).all())
        assert bool(torch.isneginf(L[0, q * B:(q + 1) * B]).all())
    check_attention(O_, Or, "O with malformed rows")
    good = np.concatenate([np.arange(q * B, (q + 1) * B) for q in range(nb) if q not in bad])
    assert np.allclose(to64(L)[0, good], Lr[0, good], atol=1e-3, rtol=0)
