"""GPU parity of the mask variants (Token Radius Attention summary, §4
ablation study: shared budget, 1D distance; Radial Attention abstract: static
window shrinking with temporal distance): radii against the oracle within fp32
rounding, CSR masks bit for bit against the oracle's brute-force block mask."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import check_csr_valid, csr_rows, need_gpu

pytestmark = pytest.mark.gpu


def run_mask(r_np, phi_np, grid, tile, bq, bk, vote, metric):
    heads, N = r_np.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    rd = torch.from_numpy(np.ascontiguousarray(r_np, np.float32)).cuda()
    phid = torch.from_numpy(np.ascontiguousarray(phi_np, np.float32)).cuda()
    ws = tra.workspace_tensor(tra.tra_mask_workspace_size(heads, grid, bq, bk, tile))
    row_ptr = torch.full((heads * (nqb + 1),), -7, dtype=torch.int32, device="cuda")
    col_idx = torch.full((heads * nqb * nkb,), -7, dtype=torch.int32, device="cuda")
    nnz = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    tra.tra_build_block_mask_ex(rd, phid, grid, bq, bk, vote, row_ptr, col_idx, nnz, ws,
                                metric, tile)
    assert tra.tra_get_device_error() == 0
    return row_ptr.cpu().numpy(), col_idx.cpu().numpy(), int(nnz.item())


def oracle_csr(r_np, phi_np, grid, tile, bq, bk, vote, metric):
    F, H, W = grid
    c = O.token_coords(F, H, W)[O.tile_major_order(F, H, W, tile)]
    masks = np.stack([O.block_mask(r_np[h], phi_np, c, bq, bk, vote, metric=metric, W=W)
                      for h in range(r_np.shape[0])])
    rp, ci = O.to_csr(masks)
    return rp.ravel(), ci


def assert_same_csr(got, ref):
    rp, ci, nnz = got
    rp_ref, ci_ref = ref
    assert nnz == len(ci_ref)
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(ci[:nnz], ci_ref)


# ---------------------------------------------------------------- radii

@pytest.mark.parametrize("wl", [workloads.TINY, workloads.WAN13B, workloads.HUNYUAN],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("budget", ["entropy", "shared"])
@pytest.mark.parametrize("metric", ["disk", "line"])
def test_radius_variants(wl, budget, metric):
    need_gpu()
    heads = min(wl.heads, 4)
    N = wl.N
    lnN = math.log(N)
    tau = 0.05
    Hs = inputs.synthetic_entropy(heads, N, wl.seed + 7, lnN - 3.0, lnN)
    if budget == "entropy":
        Hs[0, :3] = [np.inf, -np.inf, 0.0]
    else:
        Hs[heads - 1, 5] = np.inf        # one +inf entropy makes the whole head infinite
    grid = (wl.F, wl.H, wl.W)
    t_tm = O.token_coords(*grid)[O.tile_major_order(*grid, wl.tile)][:, 2]
    Hd = torch.from_numpy(Hs).cuda()
    r = torch.empty_like(Hd)
    phi = torch.empty(wl.F, dtype=torch.float32, device="cuda")
    tra.tra_budget_radius_ex(Hd, r, grid, tau, wl.gamma, budget, metric, wl.tile, phi_out=phi)
    tau32, gamma32 = float(np.float32(tau)), float(np.float32(wl.gamma))
    np.testing.assert_allclose(phi.cpu().numpy(), O.phi(np.arange(wl.F), gamma32), rtol=1e-7, atol=0)
    ref = O.radius_variant(Hs.astype(np.float64), t_tm, tau32, gamma32, wl.F, budget, metric)
    rg = r.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref)
    # entropy: fp32 table x expf; shared: evaluated in double, rounded once
    rtol = 2e-6 if budget == "entropy" else 1.2e-7
    np.testing.assert_allclose(rg[fin], ref[fin], rtol=rtol, atol=0)
    assert np.array_equal(np.isinf(rg), np.isinf(ref))
    if budget == "shared":
        assert np.isinf(rg[heads - 1]).all()
        # one radius per frame within a head
        for f in range(wl.F):
            sel = rg[0, t_tm == f]
            assert np.all(sel == sel[0])


@pytest.mark.parametrize("metric", ["disk", "line"])
def test_radial_radius(metric):
    need_gpu()
    grid = (33, 5, 6)
    r = torch.full((3, 33 * 30), -1.0, device="cuda")
    phi = torch.empty(33, dtype=torch.float32, device="cuda")
    tra.tra_radial_radius(r, grid, 7.5, metric, phi_out=phi)
    assert torch.all(r == 7.5)
    assert np.array_equal(phi.cpu().numpy(), O.radial_phi(33, metric).astype(np.float32))


# ---------------------------------------------------------------- masks

LINE_CASES = [
    # grid, tile, bq, bk, vote, radius range
    ((4, 8, 8), (1, 4, 4), 16, 16, 1, (0.2, 20.0)),
    ((4, 8, 8), (1, 4, 4), 16, 16, 5, (0.2, 20.0)),
    ((2, 6, 5), (1, 4, 4), 16, 16, 1, (0.2, 9.0)),
    ((3, 7, 9), (1, 4, 4), 16, 64, 2, (0.5, 25.0)),
    ((5, 12, 21), (1, 4, 4), 64, 64, 1, (0.3, 60.0)),
    ((5, 12, 21), (1, 4, 4), 64, 16, 16, (0.3, 60.0)),
    ((3, 17, 30), (1, 4, 4), 128, 128, 1, (0.3, 80.0)),
    ((3, 17, 30), (1, 4, 4), 128, 64, 4, (0.3, 80.0)),
    ((4, 9, 10), (2, 3, 2), 16, 64, 1, (0.3, 15.0)),
    ((6, 5, 7), (3, 2, 5), 64, 16, 3, (0.3, 15.0)),
]


@pytest.mark.parametrize("case", LINE_CASES,
                         ids=lambda c: f"{'x'.join(map(str, c[0]))}-t{''.join(map(str, c[1]))}-b{c[2]}x{c[3]}-v{c[4]}")
def test_line_mask_bitexact_small(case):
    need_gpu()
    grid, tile, bq, bk, vote, (lo, hi) = case
    F, H, W = grid
    N = F * H * W
    r = inputs.synthetic_radius(3, N, seed=N + bq + vote + 11, lo=lo, hi=hi)
    phi = O.phi(np.arange(F), 0.4).astype(np.float32)
    assert_same_csr(run_mask(r, phi, grid, tile, bq, bk, vote, "line"),
                    oracle_csr(r, phi, grid, tile, bq, bk, vote, "line"))


@pytest.mark.parametrize("metric", ["disk", "line"])
@pytest.mark.parametrize("grid,bq,vote,r0", [((15, 8, 12), 16, 1, 3.0), ((15, 8, 12), 64, 4, 5.5),
                                             ((9, 13, 11), 64, 1, 0.0), ((20, 6, 9), 16, 2, 9.0)])
def test_radial_mask_bitexact(metric, grid, bq, vote, r0):
    need_gpu()
    F, H, W = grid
    N = F * H * W
    scale = 1.0 if metric == "disk" else 4.0
    r = np.full((2, N), np.float32(r0 * scale), np.float32)
    r[1] *= np.float32(0.5)
    phi = O.radial_phi(F, metric).astype(np.float32)
    assert_same_csr(run_mask(r, phi, grid, (1, 4, 4), bq, bq, vote, metric),
                    oracle_csr(r, phi, grid, (1, 4, 4), bq, bq, vote, metric))


def test_shared_budget_mask_bitexact():
    need_gpu()
    grid, tile = (5, 12, 21), (1, 4, 4)
    F, H, W = grid
    N = F * H * W
    Hs = inputs.synthetic_entropy(3, N, 3, math.log(N) - 3.0, math.log(N))
    t_tm = O.token_coords(*grid)[O.tile_major_order(*grid, tile)][:, 2]
    r = O.radius_variant(Hs, t_tm, 0.2, 0.3, F, "shared", "disk").astype(np.float32)
    phi = O.phi(np.arange(F), 0.3).astype(np.float32)
    assert_same_csr(run_mask(r, phi, grid, tile, 64, 64, 1, "disk"),
                    oracle_csr(r, phi, grid, tile, 64, 64, 1, "disk"))


def test_line_mask_special_radii():
    need_gpu()
    grid, tile = (3, 9, 11), (1, 4, 4)
    N = 3 * 9 * 11
    phi = O.phi(np.arange(3), 0.3).astype(np.float32)
    r = np.full((2, N), np.inf, np.float32)
    r[1] = np.nan
    nqb = -(-N // 16)
    rp, ci, nnz = run_mask(r, phi, grid, tile, 16, 16, 1, "line")
    assert nnz == 2 * nqb * nqb
    r0 = np.zeros((1, N), np.float32)
    assert_same_csr(run_mask(r0, phi, grid, tile, 16, 16, 1, "line"),
                    oracle_csr(r0, phi, grid, tile, 16, 16, 1, "line"))


@pytest.mark.parametrize("wl", [workloads.WAN13B, workloads.WAN14B], ids=lambda w: w.name)
def test_line_mask_full_size_sampled(wl):
    """Full-size 1D-distance mask (all heads, the bench's launch); sampled
    query-block rows exactly against the brute-force oracle."""
    need_gpu()
    grid = (wl.F, wl.H, wl.W)
    N = wl.N
    lnN = math.log(N)
    Hs = inputs.synthetic_entropy(wl.heads, N, wl.seed + 1, lnN - 2.0, lnN)
    c = O.token_coords(*grid)[O.tile_major_order(*grid, wl.tile)]
    r = O.radius_variant(Hs, c[:, 2], 0.05, wl.gamma, wl.F, "entropy", "line").astype(np.float32)
    phi = O.phi(np.arange(wl.F), wl.gamma).astype(np.float32)
    bq, bk = wl.block_q, wl.block_k
    nqb, nkb = -(-N // bq), -(-N // bk)
    rp, ci, nnz = run_mask(r, phi, grid, wl.tile, bq, bk, 1, "line")
    check_csr_valid(rp, ci, nnz, wl.heads, nqb, nkb)
    rng = np.random.default_rng(wl.seed)
    for h in sorted({0, wl.heads - 1, int(rng.integers(wl.heads))}):
        qbs = sorted({0, nqb - 1, nqb // 2, int(rng.integers(nqb))})
        ref = O.block_mask(r[h], phi, c, bq, bk, 1, qblocks=qbs, metric="line", W=wl.W)
        for row, qb in enumerate(qbs):
            assert np.array_equal(csr_rows(rp, ci, h, qb, nqb), np.nonzero(ref[row])[0]), (h, qb)
    assert 0.0 < nnz / (wl.heads * nqb * nkb) < 1.0
