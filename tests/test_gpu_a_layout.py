"""GPU parity: tile-major permutation (bit-exact) and entropy -> radius
(within fp32 rounding) against the oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import inputs, tra, workloads
from oracle import tra_oracle as O
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

GRIDS = [((4, 8, 8), (1, 4, 4)), ((2, 6, 5), (1, 4, 4)), ((3, 7, 9), (1, 4, 4)),
         ((5, 6, 7), (2, 3, 2)), ((1, 1, 1), (1, 4, 4)), ((21, 30, 52), (1, 4, 4)),
         ((3, 45, 80), (1, 4, 4)), ((2, 13, 3), (3, 5, 7))]


@pytest.mark.parametrize("grid,tile", GRIDS, ids=lambda v: "x".join(map(str, v)))
@pytest.mark.parametrize("d", [64, 128, 8])
def test_permute_bitexact(grid, tile, d):
    need_gpu()
    F, H, W = grid
    N = F * H * W
    heads = 3
    g = torch.Generator().manual_seed(N * 7 + d)
    X = torch.randn(heads, N, d, generator=g).to(torch.bfloat16)
    pi = O.tile_major_order(F, H, W, tile)
    expect = X.view(torch.int16).numpy()
    Xd = X.cuda()
    Y = torch.empty_like(Xd)
    tra.tra_tile_major_permute(Xd, Y, grid, tile)
    got = Y.cpu().view(torch.int16).numpy()
    assert np.array_equal(got, expect[:, pi, :])
    Z = torch.empty_like(Xd)
    tra.tra_inverse_permute(Y, Z, grid, tile)
    assert torch.equal(Z, Xd)
    assert tra.tra_get_device_error() == 0


@pytest.mark.parametrize("grid,tile", GRIDS[:4], ids=lambda v: "x".join(map(str, v)))
def test_permute_f32_paths(grid, tile):
    need_gpu()
    F, H, W = grid
    N = F * H * W
    g = torch.Generator().manual_seed(N)
    X = torch.randn(2, N, 64, generator=g, dtype=torch.float32) * 3
    pi = O.tile_major_order(F, H, W, tile)
    Xd = X.cuda()
    # f32 -> bf16: round to nearest even (torch's conversion is the reference rounding)
    Yb = torch.empty(2, N, 64, dtype=torch.bfloat16, device="cuda")
    tra.tra_tile_major_permute(Xd, Yb, grid, tile)
    assert torch.equal(Yb.cpu(), X[:, pi, :].to(torch.bfloat16))
    # f32 -> f32 and back
    Yf = torch.empty_like(Xd)
    tra.tra_tile_major_permute(Xd, Yf, grid, tile)
    assert torch.equal(Yf.cpu(), X[:, pi, :])
    Zf = torch.empty_like(Xd)
    tra.tra_inverse_permute(Yf, Zf, grid, tile)
    assert torch.equal(Zf, Xd)


def test_permute_full_size_wan14b():
    """The bench's permute launch on the 21x45x80, 40-head, d=128 bf16 shape."""
    need_gpu()
    w = workloads.WAN14B
    heads = w.heads
    X = (torch.arange(heads * w.N * 8, dtype=torch.int32) % 30011).to(torch.bfloat16)
    X = X.reshape(heads, w.N, 8).repeat_interleave(16, dim=2).contiguous()
    pi = O.tile_major_order(w.F, w.H, w.W, w.tile)
    Xd = X.cuda()
    Y = torch.empty_like(Xd)
    tra.tra_tile_major_permute(Xd, Y, (w.F, w.H, w.W), w.tile)
    got = Y.cpu()
    rng = np.random.default_rng(0)
    for h in (0, heads - 1, int(rng.integers(heads))):
        assert torch.equal(got[h], X[h, torch.from_numpy(pi)])
    Z = torch.empty_like(Xd)
    tra.tra_inverse_permute(Y, Z, (w.F, w.H, w.W), w.tile)
    assert torch.equal(Z, Xd)


@pytest.mark.parametrize("wl", [workloads.TINY, workloads.WAN13B, workloads.HUNYUAN],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("tau", [4.0, 0.05])
def test_budget_radius(wl, tau):
    need_gpu()
    heads = min(wl.heads, 4)
    N = wl.N
    lnN = math.log(N)
    Hs = inputs.synthetic_entropy(heads, N, wl.seed, lnN - 3.0, lnN)
    Hs[0, :3] = [np.inf, -np.inf, 0.0]
    pi = O.tile_major_order(wl.F, wl.H, wl.W, wl.tile)
    t_tm = O.token_coords(wl.F, wl.H, wl.W)[pi][:, 2]
    Hd = torch.from_numpy(Hs).cuda()
    r = torch.empty_like(Hd)
    phi = torch.empty(wl.F, dtype=torch.float32, device="cuda")
    tra.tra_budget_radius(Hd, r, (wl.F, wl.H, wl.W), tau, wl.gamma, wl.tile, phi_out=phi)
    # the C ABI takes tau and gamma as float32: the oracle gets those same values
    tau32, gamma32 = float(np.float32(tau)), float(np.float32(wl.gamma))
    phi_ref = O.phi(np.arange(wl.F), gamma32)
    np.testing.assert_allclose(phi.cpu().numpy(), phi_ref, rtol=1e-7, atol=0)
    rg = r.cpu().numpy().astype(np.float64)
    for h in range(heads):
        ref = O.radius(Hs[h].astype(np.float64), t_tm, tau32, gamma32, wl.F, N)
        fin = np.isfinite(ref)
        np.testing.assert_allclose(rg[h][fin], ref[fin], rtol=2e-6, atol=0)
        assert np.array_equal(np.isinf(rg[h]), np.isinf(ref))
    assert rg[0, 0] == np.inf and rg[0, 1] == 0.0


@pytest.mark.parametrize("grid,tau,gamma", [((1, 8, 8), 0.05, 0.3), ((5, 8, 12), 0.05, 0.0),
                                            ((5, 8, 12), 0.05, 20.0), ((5, 8, 12), 0.0, 0.3),
                                            ((7, 4, 4), 3.0, 1.0)])
def test_budget_radius_parameter_corners(grid, tau, gamma):
    """One frame (S = 1); gamma = 0 (phi = 1, S = F); a steep decay (phi(1) ~
    2e-9); tau = 0 (every radius 0); a grid of a single tile per frame."""
    need_gpu()
    F, Hh, W = grid
    N = F * Hh * W
    heads = 3
    tile = (1, 4, 4)
    Hs = inputs.synthetic_entropy(heads, N, 11, math.log(N) - 2.0, math.log(N))
    pi = O.tile_major_order(F, Hh, W, tile)
    t_tm = O.token_coords(F, Hh, W)[pi][:, 2]
    Hd = torch.from_numpy(Hs).cuda()
    r = torch.empty_like(Hd)
    phi = torch.empty(F, dtype=torch.float32, device="cuda")
    tra.tra_budget_radius(Hd, r, grid, tau, gamma, tile, phi_out=phi)
    tau32, gamma32 = float(np.float32(tau)), float(np.float32(gamma))
    np.testing.assert_allclose(phi.cpu().numpy(), O.phi(np.arange(F), gamma32), rtol=1e-7, atol=0)
    rg = r.cpu().numpy().astype(np.float64)
    for h in range(heads):
        ref = O.radius(Hs[h].astype(np.float64), t_tm, tau32, gamma32, F, N)
        np.testing.assert_allclose(rg[h], ref, rtol=2e-6, atol=0)
    if tau == 0.0:
        assert not rg.any()
