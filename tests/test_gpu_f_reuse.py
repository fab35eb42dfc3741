"""GPU parity of the cross-step reuse loop (Token Radius Attention summary,
§2 "TRA pipeline": entropy from the dense warm-up, reused by the sparse
steps, refreshed now and then) run through the layer driver, against the
oracle's schedule: every step's output, every refreshed entropy, and the
mask every refresh builds.

The masks are compared bit for bit.  That is valid only if the GPU's entropy
(within 1e-3 of the oracle's) cannot flip a token decision, so the inputs
make every query of a head score the keys alike (identical query rows, a
per-step scale): each head then has one entropy per step and one radius per
frame, and tau is chosen so that every squared radius R^2 lies at least 0.5%
away from every squared token distance of the grid, well beyond what a 1e-3
entropy error moves it."""
import math

import numpy as np
import pytest
import torch

from entropy_adaptive_radius_b200 import tra
from entropy_adaptive_radius_b200.layer import ReusePolicy, TraLayer
from oracle import tra_oracle as O
from tests.gpu_util import H_ABS, check_attention, check_close, need_gpu, to64

pytestmark = pytest.mark.gpu

F, HH, WW, HEADS, D = 4, 8, 12, 2, 64
N = F * HH * WW
TILE = (1, 4, 4)
GAMMA = 0.35
BQ = BK = 16
SCALES = [0.5, 1.0, 2.0, 3.0, 4.5, 6.0]


def make_steps(seed):
    rng = np.random.default_rng(seed)
    u = rng.normal(size=(HEADS, 1, D))
    K0 = rng.normal(size=(HEADS, N, D))
    steps = []
    for c in SCALES:
        Q = np.broadcast_to(c * u, (HEADS, N, D))
        K = K0 + 0.05 * rng.normal(size=K0.shape)
        V = rng.normal(size=(HEADS, N, D))
        steps.append(tuple(torch.from_numpy(np.ascontiguousarray(X, np.float32)).to(torch.bfloat16)
                           for X in (Q, K, V)))
    return steps


def squared_distances():
    dx = np.arange(WW)[:, None] ** 2
    dy = np.arange(HH)[None, :] ** 2
    return np.unique((dx + dy).ravel()).astype(np.float64)


def margin(Hs, tau, c):
    """Smallest relative gap between a squared radius and a squared distance."""
    d2 = squared_distances()
    phi32 = O.phi(np.arange(F), GAMMA).astype(np.float32)
    worst = np.inf
    for H in Hs:
        for h in range(HEADS):
            r32 = O.radius(H[h], c[:, 2], tau, GAMMA, F, N).astype(np.float32)
            for t in range(F):
                rr = np.unique(r32[c[:, 2] == t])
                for dt in range(F):
                    R = (rr * phi32[dt]).astype(np.float32)
                    R2 = (R * R).astype(np.float32).astype(np.float64)
                    gap = np.min(np.abs(R2[:, None] - d2[None, :]), axis=1) / np.maximum(R2, 1.0)
                    worst = min(worst, float(gap.min()))
    return worst


def run_schedule(refresh, dtype, layout, seed=5):
    """The layer's schedule against the oracle's: outputs within the
    attention tolerances, refreshed entropies within 1e-3, and every rebuilt
    CSR bit for bit.  With layout "tile_major" the layer is handed the
    inputs already in tile-major order (permuted on the GPU once, as a model
    that keeps a transformer block's tokens in that order would) and its
    outputs are compared in that order."""
    steps = make_steps(seed=seed)
    policy = ReusePolicy(warmup=1, refresh_every=2, refresh=refresh)
    plan = O.reuse_plan(len(steps), 1, 2, refresh)
    assert [policy.kind(k) for k in range(len(steps))] == plan
    pi = O.tile_major_order(F, HH, WW, TILE)
    c = O.token_coords(F, HH, WW)[pi]
    scale = 1.0 / math.sqrt(D)
    steps_tm = [tuple(O.permute(to64(X), pi) for X in st) for st in steps]
    # entropies of the refresh steps decide the masks: pick tau with a margin
    H_ref = [O.dense_attention_entropy(*steps_tm[k], scale)[1]
             for k in range(len(steps)) if plan[k] != "sparse"]
    tau = None
    for cand in np.geomspace(0.02, 0.5, 120):
        t32 = float(np.float32(cand))
        if margin(H_ref, t32, c) > 5e-3:
            tau = t32
            break
    assert tau is not None, "no tau with a safe margin"
    gamma32 = float(np.float32(GAMMA))
    outs, used, refreshed = O.reuse_run(steps_tm, c, F, tau, gamma32, BQ, BK, 1, plan, scale)

    layer = TraLayer((F, HH, WW), HEADS, D, tau=tau, gamma=GAMMA, tile=TILE, block_q=BQ,
                     block_k=BK, policy=policy, layout=layout)
    for k, (Q, K, V) in enumerate(steps):
        if dtype == "f32":
            Q, K, V = Q.float(), K.float(), V.float()
        Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
        if layout == "tile_major":
            Og = layer(layer.to_tile_major(Qd), layer.to_tile_major(Kd), layer.to_tile_major(Vd))
            ref = outs[k]
        else:
            Og = layer(Qd, Kd, Vd)
            ref = O.inverse_permute(outs[k], pi)
        assert tra.tra_get_device_error() == 0
        check_attention(Og, ref, f"step {k} ({plan[k]}, {layout})")
        if plan[k] != "sparse":
            check_close(layer.H, refreshed[k], H_ABS, f"H step {k}")
            mask = O.mask_from_entropy(refreshed[k], c, tau, gamma32, F, BQ, BK, 1)
            rp_ref, ci_ref = O.to_csr(mask)
            nnz = int(layer.nnz.item())
            assert nnz == len(ci_ref)
            assert np.array_equal(layer.row_ptr.cpu().numpy(), rp_ref.ravel())
            assert np.array_equal(layer.col_idx[:nnz].cpu().numpy(), ci_ref)
    # the masks really change between refreshes (otherwise reuse is untested)
    refresh_steps = [k for k in range(len(steps)) if plan[k] != "sparse"]
    ms = [O.mask_from_entropy(refreshed[k], c, tau, gamma32, F, BQ, BK, 1) for k in refresh_steps]
    assert any(not np.array_equal(ms[0], m) for m in ms[1:])
    assert all(0.0 < m.mean() < 1.0 for m in ms)


@pytest.mark.parametrize("refresh,dtype", [("entropy", "bf16"), ("dense", "bf16"), ("entropy", "f32")])
def test_reuse_loop_matches_oracle_schedule(refresh, dtype):
    """dtype f32 hands the layer the same (bf16-valued) inputs as float32
    tensors: its permute then rounds them to bf16, exactly."""
    need_gpu()
    run_schedule(refresh, dtype, "original")


@pytest.mark.parametrize("refresh", ["entropy", "dense"])
def test_tile_major_resident_layer_matches_oracle_schedule(refresh):
    """The resident-layout layer (tokens kept in tile-major order between
    calls, no per-call permutes) against the oracle's schedule directly."""
    need_gpu()
    run_schedule(refresh, "bf16", "tile_major")


def test_tile_major_resident_layer_matches_original_layout():
    """layout="tile_major" runs the same kernels on already-permuted tensors:
    its outputs, permuted back, equal the original-layout layer's bit for bit,
    step by step, and so do the masks."""
    need_gpu()
    steps = make_steps(seed=8)
    policy = ReusePolicy(warmup=1, refresh_every=2, refresh="entropy")
    kw = dict(tau=0.1, gamma=GAMMA, tile=TILE, block_q=BQ, block_k=BK, policy=policy)
    a = TraLayer((F, HH, WW), HEADS, D, **kw)
    b = TraLayer((F, HH, WW), HEADS, D, layout="tile_major", **kw)
    for Q, K, V in steps:
        Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
        Oa = a(Qd, Kd, Vd)
        Ob_tm = b(b.to_tile_major(Qd), b.to_tile_major(Kd), b.to_tile_major(Vd))
        assert torch.equal(b.from_tile_major(Ob_tm), Oa)
        assert int(a.nnz.item()) == int(b.nnz.item())
        assert torch.equal(a.row_ptr, b.row_ptr)
    assert tra.tra_get_device_error() == 0
    with pytest.raises(ValueError):
        TraLayer((F, HH, WW), HEADS, D, layout="diagonal", **kw)


@pytest.mark.parametrize("budget,metric,r0", [("shared", "disk", None), ("entropy", "line", None),
                                              ("entropy", "disk", 2.5), ("entropy", "line", 9.0)])
def test_layer_mask_variants_match_the_component_calls(budget, metric, r0):
    """The layer's variant masks are the ones the variant entry points build
    from its own entropy (the components are pinned to the oracle in
    test_gpu_d_variants); the sparse steps then use them."""
    need_gpu()
    steps = make_steps(seed=11)
    layer = TraLayer((F, HH, WW), HEADS, D, tau=0.1, gamma=GAMMA, tile=TILE, block_q=BQ, block_k=BK,
                     budget=budget, metric=metric, radial_r0=r0)
    Q, K, V = (x.cuda() for x in steps[0])
    layer(Q, K, V)
    grid = (F, HH, WW)
    r = torch.empty_like(layer.H)
    phi = torch.empty(F, dtype=torch.float32, device="cuda")
    if r0 is None:
        tra.tra_budget_radius_ex(layer.H, r, grid, 0.1, GAMMA, budget, metric, TILE, phi_out=phi)
    else:
        tra.tra_radial_radius(r, grid, r0, metric, TILE, phi_out=phi)
    nqb = -(-N // BQ)
    rp = torch.empty(HEADS * (nqb + 1), dtype=torch.int32, device="cuda")
    ci = torch.empty(HEADS * nqb * nqb, dtype=torch.int32, device="cuda")
    nnz = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = tra.workspace_tensor(tra.tra_mask_workspace_size(HEADS, grid, BQ, BK, TILE))
    tra.tra_build_block_mask_ex(r, phi, grid, BQ, BK, 1, rp, ci, nnz, ws, metric, TILE)
    n = int(nnz.item())
    assert n == int(layer.nnz.item()) and torch.equal(rp, layer.row_ptr)
    assert torch.equal(ci[:n], layer.col_idx[:n])
    O1 = layer(*(x.cuda() for x in steps[1]))            # a sparse step over that mask
    assert tra.tra_get_device_error() == 0 and bool(torch.isfinite(O1.float()).all())
