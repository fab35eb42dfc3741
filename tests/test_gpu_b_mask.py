"""GPU parity of the fused radius mask: the CSR must equal the oracle's
brute-force block mask bit for bit, given the same fp32 radii and phi table."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import check_csr_valid, csr_rows, need_gpu

pytestmark = pytest.mark.gpu


def run_mask(r_np, phi_np, grid, tile, bq, bk, vote, capacity=None):
    heads, N = r_np.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    rd = torch.from_numpy(np.ascontiguousarray(r_np, np.float32)).cuda()
    phid = torch.from_numpy(np.ascontiguousarray(phi_np, np.float32)).cuda()
    ws = tra.workspace_tensor(tra.tra_mask_workspace_size(heads, grid, bq, bk, tile))
    row_ptr = torch.full((heads * (nqb + 1),), -7, dtype=torch.int32, device="cuda")
    cap = heads * nqb * nkb if capacity is None else capacity
    col_idx = torch.full((max(cap, 1),), -7, dtype=torch.int32, device="cuda")[:cap]
    nnz = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    tra.tra_build_block_mask(rd, phid, grid, bq, bk, vote, row_ptr, col_idx, nnz, ws, tile)
    assert tra.tra_get_device_error() == 0
    return row_ptr.cpu().numpy(), col_idx.cpu().numpy(), int(nnz.item())


def oracle_csr(r_np, phi_np, grid, tile, bq, bk, vote):
    F, H, W = grid
    pi = O.tile_major_order(F, H, W, tile)
    c = O.token_coords(F, H, W)[pi]
    masks = np.stack([O.block_mask(r_np[h], phi_np, c, bq, bk, vote) for h in range(r_np.shape[0])])
    rp, ci = O.to_csr(masks)
    return rp.ravel(), ci, masks


CASES = [
    # grid, tile, bq, bk, vote, radius range
    ((4, 8, 8), (1, 4, 4), 16, 16, 1, (0.2, 6.0)),
    ((4, 8, 8), (1, 4, 4), 16, 16, 4, (0.2, 6.0)),
    ((4, 8, 8), (1, 4, 4), 16, 16, 16, (0.2, 6.0)),
    ((2, 6, 5), (1, 4, 4), 16, 16, 1, (0.2, 3.0)),
    ((3, 7, 9), (1, 4, 4), 16, 64, 2, (0.5, 5.0)),
    ((5, 12, 21), (1, 4, 4), 64, 64, 1, (0.3, 8.0)),
    ((5, 12, 21), (1, 4, 4), 64, 16, 16, (0.3, 8.0)),
    ((3, 17, 30), (1, 4, 4), 128, 128, 1, (0.3, 10.0)),
    ((3, 17, 30), (1, 4, 4), 128, 64, 4, (0.3, 10.0)),
    ((4, 9, 10), (2, 3, 2), 16, 64, 1, (0.3, 5.0)),
    ((6, 5, 7), (3, 2, 5), 64, 16, 3, (0.3, 5.0)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{'x'.join(map(str, c[0]))}-t{''.join(map(str, c[1]))}-b{c[2]}x{c[3]}-v{c[4]}")
def test_mask_bitexact_small(case):
    need_gpu()
    grid, tile, bq, bk, vote, (lo, hi) = case
    F, H, W = grid
    N = F * H * W
    heads = 3
    r = inputs.synthetic_radius(heads, N, seed=N + bq + vote, lo=lo, hi=hi)
    phi = O.phi(np.arange(F), 0.4).astype(np.float32)
    rp, ci, nnz = run_mask(r, phi, grid, tile, bq, bk, vote)
    rp_ref, ci_ref, _ = oracle_csr(r, phi, grid, tile, bq, bk, vote)
    assert nnz == len(ci_ref)
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(ci[:nnz], ci_ref)


def test_mask_tiny_workload():
    """The tiny workload's mask (tau = 4, gamma = 0.5, vote 1) from radii of
    spread-out entropies; also the brute-force superset property."""
    need_gpu()
    w = workloads.TINY
    grid = (w.F, w.H, w.W)
    H = inputs.synthetic_entropy(w.heads, w.N, 0, math.log(w.N) - 4, math.log(w.N))
    pi = O.tile_major_order(*grid, w.tile)
    c = O.token_coords(*grid)[pi]
    r = np.stack([O.radius(H[h], c[:, 2], 0.25, w.gamma, w.F, w.N) for h in range(w.heads)]).astype(np.float32)
    phi = O.phi(np.arange(w.F), w.gamma).astype(np.float32)
    rp, ci, nnz = run_mask(r, phi, grid, w.tile, 16, 16, 1)
    rp_ref, ci_ref, masks = oracle_csr(r, phi, grid, w.tile, 16, 16, 1)
    assert np.array_equal(rp, rp_ref) and np.array_equal(ci[:nnz], ci_ref)
    for h in range(w.heads):
        M = O.token_mask(r[h], phi, c, c)
        qi, kj = np.nonzero(M)
        assert masks[h][qi // 16, kj // 16].all()


def test_mask_infinite_radius_is_dense_and_overflow_reports_nnz():
    need_gpu()
    grid, tile = (3, 9, 11), (1, 4, 4)
    N = 3 * 9 * 11
    r = np.full((2, N), np.inf, np.float32)
    phi = O.phi(np.arange(3), 0.3).astype(np.float32)
    nqb = nkb = -(-N // 16)
    rp, ci, nnz = run_mask(r, phi, grid, tile, 16, 16, 1)
    assert nnz == 2 * nqb * nkb
    assert np.array_equal(ci[:nnz], np.tile(np.arange(nkb), 2 * nqb))
    # capacity too small: nnz still reports the full count, the prefix is right
    rp2, ci2, nnz2 = run_mask(r, phi, grid, tile, 16, 16, 1, capacity=50)
    assert nnz2 == nnz and np.array_equal(rp2, rp) and np.array_equal(ci2[:50], ci[:50])


def test_mask_monotone_in_radius_and_vote():
    need_gpu()
    grid, tile = (4, 20, 24), (1, 4, 4)
    N = 4 * 20 * 24
    r = inputs.synthetic_radius(2, N, seed=5, lo=0.5, hi=6.0, special=False)
    phi = O.phi(np.arange(4), 0.3).astype(np.float32)
    nqb = nkb = -(-N // 64)

    def dense(rr, v):
        rp, ci, nnz = run_mask(rr, phi, grid, tile, 64, 64, v)
        m = np.zeros((2, nqb, nkb), bool)
        for h in range(2):
            for qb in range(nqb):
                m[h, qb, csr_rows(rp, ci, h, qb, nqb)] = True
        return m

    base = dense(r, 1)
    assert np.all(dense(r * np.float32(1.5), 1) >= base)
    prev = base
    for v in (2, 8, 64, 512):
        cur = dense(r, v)
        assert np.all(cur <= prev)
        prev = cur


@pytest.mark.parametrize("wl,vote", [(workloads.WAN13B, 1), (workloads.WAN14B, 1),
                                     (workloads.WAN14B, 16), (workloads.HUNYUAN, 1)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_mask_full_size_sampled(wl, vote):
    """Full-size mask launch (all heads, as the bench runs it); sampled query
    block rows compared exactly with the brute-force oracle, the rest checked
    for CSR validity and the diagonal property."""
    need_gpu()
    grid = (wl.F, wl.H, wl.W)
    N = wl.N
    lnN = math.log(N)
    Hs = inputs.synthetic_entropy(wl.heads, N, wl.seed, lnN - 2.0, lnN)
    pi = O.tile_major_order(*grid, wl.tile)
    c = O.token_coords(*grid)[pi]
    r = np.stack([O.radius(Hs[h], c[:, 2], 0.05, wl.gamma, wl.F, N) for h in range(wl.heads)]).astype(np.float32)
    phi = O.phi(np.arange(wl.F), wl.gamma).astype(np.float32)
    bq, bk = wl.block_q, wl.block_k
    nqb, nkb = -(-N // bq), -(-N // bk)
    rp, ci, nnz = run_mask(r, phi, grid, wl.tile, bq, bk, vote)
    check_csr_valid(rp, ci, nnz, wl.heads, nqb, nkb)
    rng = np.random.default_rng(wl.seed)
    for h in sorted({0, wl.heads - 1, int(rng.integers(wl.heads))}):
        qbs = sorted({0, nqb - 1, nqb // 2, int(rng.integers(nqb))})
        ref = O.block_mask(r[h], phi, c, bq, bk, vote, qblocks=qbs)
        for row, qb in enumerate(qbs):
            got = csr_rows(rp, ci, h, qb, nqb)
            assert np.array_equal(got, np.nonzero(ref[row])[0]), (h, qb)
    if vote <= bq:
        # every query lies in its own disk: when |qb| = |kb| the diagonal block
        # collects >= |qb| votes
        if bq == bk:
            for h in range(wl.heads):
                for qb in range(0, nqb, max(1, nqb // 17)):
                    if vote <= min(bq, N - qb * bq):
                        assert qb in set(csr_rows(rp, ci, h, qb, nqb).tolist())
    kept = nnz / (wl.heads * nqb * nkb)
    assert 0.0 < kept < 1.0


@pytest.mark.parametrize("grid,tile,bq,bk,vote", [((1, 9, 13), (1, 4, 4), 16, 16, 1),
                                                  ((384, 4, 4), (1, 4, 4), 16, 16, 20),
                                                  ((384, 4, 4), (2, 4, 4), 64, 16, 70)])
def test_mask_frame_count_extremes(grid, tile, bq, bk, vote):
    """One frame, and the largest frame count the mask accepts (its per-frame
    threshold table then needs the opt-in shared-memory size).  Every query
    keeps its own (x, y) in every frame, so with many small frames the vote
    threshold is set above those self votes to make the mask non-trivial."""
    need_gpu()
    F, H, W = grid
    N = F * H * W
    r = inputs.synthetic_radius(2, N, seed=F + bq, lo=0.3, hi=3.0, special=False)
    phi = O.phi(np.arange(F), 0.6).astype(np.float32)
    rp, ci, nnz = run_mask(r, phi, grid, tile, bq, bk, vote)
    rp_ref, ci_ref, _ = oracle_csr(r, phi, grid, tile, bq, bk, vote)
    assert nnz == len(ci_ref)
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(ci[:nnz], ci_ref)
    assert 0.0 < nnz / (2 * (-(-N // bq)) * (-(-N // bk))) < 1.0


@pytest.mark.parametrize("vote,hi", [(257, 3.0), (40, 2.5)])
def test_mask_with_empty_rows_drives_attention(vote, hi):
    """A vote threshold above |qb| * |kb| keeps nothing (nnz = 0, every CSR row
    empty); one above the self votes with small radii empties some rows.  The
    CSR matches the oracle bit for bit, and the block-sparse call over it gives
    O = 0 and LSE = -inf on the empty rows and the oracle's attention on the
    others."""
    need_gpu()
    grid, tile, B = (4, 8, 8), (1, 4, 4), 16
    F, H, W = grid
    N = F * H * W
    heads = 2
    r = inputs.synthetic_radius(heads, N, seed=vote, lo=0.2, hi=hi, special=False)
    phi = O.phi(np.arange(F), 0.4).astype(np.float32)
    rp, ci, nnz = run_mask(r, phi, grid, tile, B, B, vote)
    rp_ref, ci_ref, masks = oracle_csr(r, phi, grid, tile, B, B, vote)
    assert nnz == len(ci_ref) and np.array_equal(rp, rp_ref) and np.array_equal(ci[:nnz], ci_ref)
    empty = ~masks.any(axis=2)
    if vote > B * B:
        assert nnz == 0 and empty.all()
    else:
        assert empty.any() and not empty.all()
    g = torch.Generator().manual_seed(vote)
    Q, K, V = (torch.randn(heads, N, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    Os = torch.full((heads, N, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    Ls = torch.empty(heads, N, dtype=torch.float32, device="cuda")
    ci_d = torch.from_numpy(ci[:max(nnz, 1)] if nnz else np.zeros(1, np.int32)).cuda()
    tra.tra_block_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), Os, torch.from_numpy(rp).cuda(), ci_d,
                              B, B, lse=Ls)
    assert tra.tra_get_device_error() == 0
    Or, Lr = O.sparse_attention(Q.double().numpy(), K.double().numpy(), V.double().numpy(), masks,
                                B, B, 1.0 / math.sqrt(64))
    rows_empty = np.repeat(empty, B, axis=1)[:, :N]
    Osn, Lsn = Os.float().cpu().numpy(), Ls.cpu().numpy()
    assert (Osn[rows_empty] == 0).all() and np.isneginf(Lsn[rows_empty]).all()
    assert np.abs(Osn - Or).max() <= 2e-2 and np.abs(Osn - Or).mean() <= 2e-3
    keep = ~rows_empty
    if keep.any():
        assert np.abs(Lsn[keep] - Lr[keep]).max() <= 1e-3
