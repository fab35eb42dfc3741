"""Pins of the oracle's cross-step reuse schedule (CPU): hand-written plans,
and schedules that reduce to the pinned dense / sparse attention; plus the
host-side step sequencing of the layer driver against the oracle's plan."""

import numpy as np
import pytest

from entropy_adaptive_radius_b200.layer import ReusePolicy
from oracle import tra_oracle as O


def test_reuse_plan_hand_written():
    assert O.reuse_plan(5, 1, 0, "entropy") == ["dense"] + ["sparse"] * 4
    assert O.reuse_plan(8, 1, 3, "entropy") == ["dense", "sparse", "sparse", "sparse+entropy",
                                                "sparse", "sparse", "sparse+entropy", "sparse"]
    assert O.reuse_plan(7, 2, 2, "dense") == ["dense", "dense", "sparse", "dense", "sparse",
                                              "dense", "sparse"]
    assert O.reuse_plan(3, 1, 1, "dense") == ["dense"] * 3


@pytest.mark.parametrize("steps,warmup,every,refresh",
                         [(10, 1, 0, "entropy"), (12, 1, 4, "entropy"), (9, 3, 2, "dense"),
                          (50, 5, 10, "entropy"), (6, 1, 1, "entropy"), (20, 2, 7, "dense")])
def test_layer_policy_matches_oracle_plan(steps, warmup, every, refresh):
    pol = ReusePolicy(warmup=warmup, refresh_every=every, refresh=refresh)
    assert [pol.kind(k) for k in range(steps)] == O.reuse_plan(steps, warmup, every, refresh)


def test_layer_policy_rejects_bad_settings():
    with pytest.raises(ValueError):
        ReusePolicy(warmup=0)
    with pytest.raises(ValueError):
        ReusePolicy(refresh="never")
    with pytest.raises(ValueError):
        ReusePolicy(refresh_every=-1)


def _steps(F, H, W, heads, d, n, seed):
    rng = np.random.default_rng(seed)
    pi = O.tile_major_order(F, H, W, (1, 4, 4))
    out = []
    for _ in range(n):
        Q = rng.normal(size=(heads, F * H * W, d)) * 0.7
        K = rng.normal(size=(heads, F * H * W, d))
        V = rng.normal(size=(heads, F * H * W, d))
        out.append(tuple(O.permute(X, pi) for X in (Q, K, V)))
    return out, O.token_coords(F, H, W)[pi]


def test_all_dense_schedule_is_dense_attention():
    F, H, W, heads, d = 2, 4, 8, 2, 16
    steps, c = _steps(F, H, W, heads, d, 3, seed=0)
    plan = O.reuse_plan(3, 1, 1, "dense")
    outs, used, refreshed = O.reuse_run(steps, c, F, 0.5, 0.3, 16, 16, 1, plan, 0.25)
    for k, (Q, K, V) in enumerate(steps):
        Od, Hd, _ = O.dense_attention_entropy(Q, K, V, 0.25)
        assert np.array_equal(outs[k], Od)
        assert np.array_equal(refreshed[k], Hd)
        assert used[k] is None


def test_huge_budget_sparse_steps_equal_dense():
    # tau so large that every radius covers the grid: every block is kept and
    # the sparse steps reduce to dense attention
    F, H, W, heads, d = 2, 4, 8, 2, 16
    steps, c = _steps(F, H, W, heads, d, 4, seed=1)
    plan = O.reuse_plan(4, 1, 2, "entropy")
    outs, used, _ = O.reuse_run(steps, c, F, 1e6, 0.3, 16, 16, 1, plan, 0.25)
    for k, (Q, K, V) in enumerate(steps):
        Od, _, _ = O.dense_attention_entropy(Q, K, V, 0.25)
        assert np.allclose(outs[k], Od, rtol=0, atol=1e-12)
        if k > 0:
            assert used[k].all()


def test_refresh_uses_this_steps_entropy_for_the_next_steps():
    F, H, W, heads, d = 3, 4, 8, 2, 16
    steps, c = _steps(F, H, W, heads, d, 5, seed=2)
    plan = O.reuse_plan(5, 1, 2, "entropy")          # dense, sparse, sparse+entropy, sparse, sparse+entropy
    tau, gamma = 0.3, 0.5
    outs, used, refreshed = O.reuse_run(steps, c, F, tau, gamma, 16, 16, 1, plan, 0.25)
    H0 = O.dense_attention_entropy(*steps[0], 0.25)[1]
    H2 = O.dense_attention_entropy(*steps[2], 0.25)[1]
    m0 = O.mask_from_entropy(H0, c, tau, gamma, F, 16, 16, 1)
    m2 = O.mask_from_entropy(H2, c, tau, gamma, F, 16, 16, 1)
    assert np.array_equal(used[1], m0) and np.array_equal(used[2], m0)
    assert np.array_equal(used[3], m2) and np.array_equal(used[4], m2)
    assert np.array_equal(refreshed[2], H2) and set(refreshed) == {0, 2, 4}
    # the refresh step's own output still uses the old mask
    O2, _ = O.sparse_attention(*steps[2], m0, 16, 16, 0.25)
    assert np.array_equal(outs[2], O2)
