"""Pins of the CPU oracle against facts fixed outside the oracle itself:
hand-written orders, textbook lattice counts, closed forms, a library
attention routine, and brute-force enumeration on tiny inputs."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import tra_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_orders():
    cases = []
    with open(os.path.join(GOLDEN, "tile_major_orders.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, tail = line.split(":")
            F, H, W, tt, ty, tx = map(int, head.split())
            cases.append(((F, H, W), (tt, ty, tx), [int(v) for v in tail.split()]))
    return cases


# --------------------------------------------------------------------------
# tile-major permutation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden_orders(), ids=lambda c: "x".join(map(str, c[0])))
def test_tile_major_matches_hand_written(case):
    (F, H, W), tile, expected = case
    assert O.tile_major_order(F, H, W, tile).tolist() == expected


@pytest.mark.parametrize("grid,tile", [((4, 8, 8), (1, 4, 4)), ((3, 7, 9), (1, 4, 4)),
                                       ((5, 6, 7), (2, 3, 2)), ((21, 30, 52), (1, 4, 4)),
                                       ((2, 1, 1), (1, 4, 4))])
def test_tile_major_is_bijection_and_inverse(grid, tile):
    F, H, W = grid
    pi = O.tile_major_order(F, H, W, tile)
    N = F * H * W
    assert sorted(pi.tolist()) == list(range(N))
    X = np.arange(2 * N * 3, dtype=np.float64).reshape(2, N, 3)
    assert np.array_equal(O.inverse_permute(O.permute(X, pi), pi), X)


def test_tile_major_keeps_tiles_contiguous():
    # every run of 16 positions of a 4x4 tiling of a 8x12 frame is one 4x4 square
    pi = O.tile_major_order(1, 8, 12, (1, 4, 4))
    c = O.token_coords(1, 8, 12)[pi]
    for s in range(0, 96, 16):
        xs, ys = c[s:s + 16, 0], c[s:s + 16, 1]
        assert xs.max() - xs.min() == 3 and ys.max() - ys.min() == 3


# --------------------------------------------------------------------------
# entropy
# --------------------------------------------------------------------------

def test_uniform_scores_give_log_n():
    N, d = 300, 16
    rng = np.random.default_rng(0)
    K = rng.standard_normal((N, d))
    Q = np.zeros((5, d))
    _, L, P = O.softmax_attention(Q, K, K, 1.0 / math.sqrt(d))
    H = O.entropy_from_probs(P)
    np.testing.assert_allclose(H, math.log(N), atol=1e-12)
    np.testing.assert_allclose(O.entropy_from_scores(O.scores(Q, K, 0.25)), math.log(N), atol=1e-12)
    np.testing.assert_allclose(L, math.log(N), atol=1e-12)


def test_one_hot_row_gives_zero_entropy():
    d = 8
    K = np.zeros((10, d))
    K[3, 0] = 1.0
    Q = np.zeros((1, d))
    Q[0, 0] = 4000.0           # score gap 4000 / sqrt(8) > 1100: other weights underflow to 0
    _, _, P = O.softmax_attention(Q, K, K, 1.0 / math.sqrt(d))
    assert P[0, 3] == 1.0
    assert O.entropy_from_probs(P)[0] == 0.0
    assert abs(O.entropy_from_scores(O.scores(Q, K, 1.0 / math.sqrt(d)))[0]) < 1e-12


@pytest.mark.parametrize("p", [0.5, 0.1, 0.9, 0.01])
def test_two_point_distribution_closed_form(p):
    # scores ln p, ln(1-p) give the binary entropy -p ln p - (1-p) ln(1-p)
    s = np.array([[math.log(p), math.log(1 - p)]])
    expect = -p * math.log(p) - (1 - p) * math.log(1 - p)
    assert abs(O.entropy_from_scores(s)[0] - expect) < 1e-14
    e = np.exp(s)
    assert abs(O.entropy_from_probs(e / e.sum())[0] - expect) < 1e-14


def test_entropy_forms_agree_and_bounded():
    rng = np.random.default_rng(1)
    s = rng.standard_normal((50, 200)) * rng.uniform(0.1, 10, size=(50, 1))
    H1 = O.entropy_from_scores(s)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    H2 = O.entropy_from_probs(e / e.sum(axis=1, keepdims=True))
    np.testing.assert_allclose(H1, H2, atol=1e-11)
    assert np.all(H1 >= -1e-12) and np.all(H1 <= math.log(200) + 1e-12)


# --------------------------------------------------------------------------
# attention against a library routine
# --------------------------------------------------------------------------

def _sdpa(Q, K, V, mask=None):
    q, k, v = (torch.from_numpy(np.asarray(a, np.float64))[None] for a in (Q, K, V))
    m = None if mask is None else torch.from_numpy(mask)[None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)[0].numpy()


def test_dense_attention_matches_library_sdpa():
    rng = np.random.default_rng(2)
    Q, K, V = (rng.standard_normal((2, 77, 24)) for _ in range(3))
    Q *= 3
    Oo, H, L = O.dense_attention_entropy(Q, K, V, 1.0 / math.sqrt(24))
    for h in range(2):
        np.testing.assert_allclose(Oo[h], _sdpa(Q[h], K[h], V[h]), atol=1e-12)
        s = Q[h] @ K[h].T / math.sqrt(24)
        np.testing.assert_allclose(L[h], np.log(np.exp(s).sum(axis=1)), atol=1e-12)
        np.testing.assert_allclose(H[h], O.entropy_from_scores(s), atol=1e-11)


def test_sparse_attention_matches_library_masked_sdpa():
    rng = np.random.default_rng(3)
    N, d, B = 70, 16, 16
    Q, K, V = (rng.standard_normal((1, N, d)) for _ in range(3))
    nb = -(-N // B)
    mask = rng.random((1, nb, nb)) < 0.4
    mask[0, np.arange(nb), np.arange(nb)] = True
    Os, _ = O.sparse_attention(Q, K, V, mask, B, B, 1.0 / math.sqrt(d))
    tok = np.repeat(np.repeat(mask[0], B, axis=0), B, axis=1)[:N, :N]
    np.testing.assert_allclose(Os[0], _sdpa(Q[0], K[0], V[0], tok), atol=1e-12)


def test_sparse_all_ones_equals_dense_and_empty_row_is_zero():
    rng = np.random.default_rng(4)
    N, d = 50, 8
    Q, K, V = (rng.standard_normal((1, N, d)) for _ in range(3))
    full = np.ones((1, 4, 4), bool)
    Os, Ls = O.sparse_attention(Q, K, V, full, 16, 16, 0.3)
    Od, _, Ld = O.dense_attention_entropy(Q, K, V, 0.3)
    np.testing.assert_allclose(Os, Od, atol=1e-13)
    np.testing.assert_allclose(Ls, Ld, atol=1e-13)
    empty = full.copy()
    empty[0, 1, :] = False
    Oe, Le = O.sparse_attention(Q, K, V, empty, 16, 16, 0.3)
    assert np.all(Oe[0, 16:32] == 0) and np.all(Le[0, 16:32] == -np.inf)


# --------------------------------------------------------------------------
# budget, decay, radius
# --------------------------------------------------------------------------

def test_budget_at_uniform_entropy_is_tau():
    for N in (256, 32760, 75600):
        for tau in (0.01, 0.5, 4.0):
            assert abs(O.budget(math.log(N), tau, N) - tau) < 1e-12 * max(1, tau)


def test_frame_energy_closed_form():
    # sum_{t'} exp(-2 gamma |t'-t|) as two finite geometric series
    for F, g in ((1, 0.3), (4, 0.5), (21, 0.3), (33, 0.2), (7, 0.0)):
        S = O.frame_energy(F, g)
        q = math.exp(-2 * g)
        for t in range(F):
            if q == 1.0:
                expect = F
            else:
                expect = (1 - q ** (t + 1)) / (1 - q) + q * (1 - q ** (F - 1 - t)) / (1 - q)
            assert abs(S[t] - expect) < 1e-12


def test_phi_values():
    assert O.phi(0, 0.3) == 1.0
    assert abs(O.phi(2, 0.5) - math.exp(-1.0)) < 1e-15
    assert abs(O.phi(10, 0.2) / O.phi(9, 0.2) - math.exp(-0.2)) < 1e-14


def _disk_counts():
    out = {}
    with open(os.path.join(GOLDEN, "lattice_disk_counts.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                n, c = map(int, line.split())
                out[n] = c
    return out


def test_token_mask_disk_counts_match_lattice_counts():
    counts = _disk_counts()
    F, H, W = 1, 21, 21
    ck = O.token_coords(F, H, W)
    cq = np.array([[10, 10, 0]])
    phi32 = np.ones(1, np.float32)
    for n, c in counts.items():
        r = np.float32(math.sqrt(n) + 1e-4)        # just above sqrt(n): R2 in [n, n + 1)
        M = O.token_mask(np.array([r]), phi32, cq, ck)
        assert M.sum() == c, (n, M.sum(), c)
    # radii that are exact integers put lattice points exactly on the circle:
    # the compare is inclusive, so they count
    for k in (1, 2, 3, 4):
        M = O.token_mask(np.array([np.float32(k)]), phi32, cq, ck)
        assert M.sum() == counts[k * k]


def test_token_mask_temporal_decay_is_symmetric_and_shrinks():
    F, H, W = 9, 25, 25
    ck = O.token_coords(F, H, W)
    cq = np.array([[12, 12, 4]])
    gamma = 0.3
    phi32 = O.phi(np.arange(F), gamma).astype(np.float32)
    r = np.array([8.0], np.float32)
    M = O.token_mask(r, phi32, cq, ck).reshape(F, H * W).sum(axis=1)
    for delta in range(1, 5):
        assert M[4 - delta] == M[4 + delta]
        assert M[4 + delta] <= M[4 + delta - 1]
        # count equals the lattice count of the disk of radius r * phi(delta)
        R2 = float(np.float32(np.float32(8.0 * phi32[delta]) ** 2))
        dx = np.arange(-13, 14)
        brute = int(((dx[:, None] ** 2 + dx[None, :] ** 2) <= R2).sum())
        assert M[4 + delta] == brute


def test_token_mask_special_radii():
    F, H, W = 3, 5, 6
    ck = O.token_coords(F, H, W)
    cq = np.array([[2, 1, 1], [0, 0, 0], [5, 4, 2]])
    phi32 = O.phi(np.arange(F), 0.5).astype(np.float32)
    r = np.array([np.inf, np.nan, 0.0], np.float32)
    M = O.token_mask(r, phi32, cq, ck)
    assert M[0].all() and M[1].all()
    # r = 0: only keys at the query's own (x, y), one per frame
    assert M[2].sum() == F
    assert np.all(ck[M[2]][:, :2] == [5, 4])


def test_radius_budget_conservation_far_from_edges():
    # a query in the middle of a large grid: the disks of all frames together hold
    # about K = tau * e^H tokens (equal-area reading), up to the lattice error
    F, H, W = 5, 121, 121
    gamma, tau = 0.3, 0.5
    N = F * H * W
    Hq = np.array([math.log(N) - 1.0])
    t_q = 2
    r = O.radius(Hq, [t_q], tau, gamma, F, N)
    K = tau * math.exp(Hq[0])
    phi32 = O.phi(np.arange(F), gamma).astype(np.float32)
    ck = O.token_coords(F, H, W)
    M = O.token_mask(r.astype(np.float32), phi32, np.array([[60, 60, t_q]]), ck)
    Rsum = sum(float(r[0]) * math.exp(-gamma * abs(t - t_q)) for t in range(F))
    assert abs(M.sum() - K) <= 4 * Rsum + 4 * F, (M.sum(), K)
    # the exact area identity behind it
    assert abs(math.pi * r[0] ** 2 * O.frame_energy(F, gamma)[t_q] - K) < 1e-9 * K


# --------------------------------------------------------------------------
# block votes, block mask, CSR
# --------------------------------------------------------------------------

def _tiny_setup(seed=0):
    F, H, W = 4, 8, 8
    pi = O.tile_major_order(F, H, W, (1, 4, 4))
    c = O.token_coords(F, H, W)[pi]
    rng = np.random.default_rng(seed)
    r = rng.uniform(0.0, 4.0, size=F * H * W).astype(np.float32)
    phi32 = O.phi(np.arange(F), 0.5).astype(np.float32)
    return c, r, phi32


def test_block_votes_brute_force():
    c, r, phi32 = _tiny_setup()
    M = O.token_mask(r, phi32, c, c)
    votes = O.block_votes(M, 16, 16)
    for qb in (0, 5, 15):
        for kb in (0, 7, 15):
            n = 0
            for i in range(qb * 16, qb * 16 + 16):
                for j in range(kb * 16, kb * 16 + 16):
                    dx, dy, dt = c[i, 0] - c[j, 0], c[i, 1] - c[j, 1], abs(c[i, 2] - c[j, 2])
                    R = np.float32(r[i] * phi32[dt])
                    n += int(dx * dx + dy * dy <= float(np.float32(R * R)))
            assert votes[qb, kb] == n


def test_block_mask_superset_of_token_mask_at_vote_one():
    c, r, phi32 = _tiny_setup(1)
    M = O.token_mask(r, phi32, c, c)
    bm = O.block_mask(r, phi32, c, 16, 16, 1)
    qi, kj = np.nonzero(M)
    assert bm[qi // 16, kj // 16].all()
    # and every kept block holds at least one token pair
    votes = O.block_votes(M, 16, 16)
    assert np.array_equal(bm, votes >= 1)


def test_block_mask_infinite_radius_all_ones_and_monotone():
    c, r, phi32 = _tiny_setup(2)
    assert O.block_mask(np.full_like(r, np.inf), phi32, c, 16, 16, 1).all()
    small = O.block_mask(r * np.float32(0.5), phi32, c, 16, 16, 1)
    big = O.block_mask(r, phi32, c, 16, 16, 1)
    assert np.all(big >= small)
    prev = None
    for v in (1, 2, 4, 16, 64, 256):
        cur = O.block_mask(r, phi32, c, 16, 16, v)
        if prev is not None:
            assert np.all(cur <= prev)
        prev = cur
    # diagonal blocks hold >= 16 self votes (every query is inside its own disk)
    assert O.block_mask(r, phi32, c, 16, 16, 16).diagonal().all()


def test_block_mask_ragged_blocks():
    F, H, W = 2, 6, 5
    pi = O.tile_major_order(F, H, W, (1, 4, 4))
    c = O.token_coords(F, H, W)[pi]
    r = np.full(60, 1.0, np.float32)
    phi32 = O.phi(np.arange(F), 0.5).astype(np.float32)
    bm = O.block_mask(r, phi32, c, 16, 16, 1)
    assert bm.shape == (4, 4)
    M = O.token_mask(r, phi32, c, c)
    assert np.array_equal(bm, O.block_votes(M, 16, 16) >= 1)


def test_csr_definition():
    m = np.array([[[1, 0, 1], [0, 0, 0]], [[0, 1, 0], [1, 1, 1]]], bool)
    row_ptr, col = O.to_csr(m)
    assert row_ptr.tolist() == [[0, 2, 2], [2, 3, 6]]
    assert col.tolist() == [0, 2, 1, 0, 1, 2]
