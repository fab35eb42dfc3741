"""Pins of the oracle's mask variants (CPU only): the shared-budget and
1D-distance ablations (Token Radius Attention summary, §4 ablation study) and
the static shrinking window of Radial Attention (abstract).  Each check comes
from outside the oracle: a closed form, a hand-worked example, a special case
that reduces to the pinned entropy-budget disk, or the growth law the Radial
page states (support that grows with log F)."""
import math

import numpy as np
import pytest

from oracle import tra_oracle as O


def test_frame_length_closed_form():
    # sum_{t'} exp(-gamma |t'-t|) as two finite geometric series
    for F, g in ((1, 0.3), (4, 0.5), (21, 0.3), (33, 0.2), (6, 0.0)):
        L = O.frame_length(F, g)
        q = math.exp(-g)
        for t in range(F):
            expect = F if q == 1.0 else (1 - q ** (t + 1)) / (1 - q) + q * (1 - q ** (F - 1 - t)) / (1 - q)
            assert abs(L[t] - expect) < 1e-12


@pytest.mark.parametrize("metric", ["disk", "line"])
def test_shared_budget_with_constant_entropy_is_the_entropy_budget(metric):
    F, N, heads = 5, 200, 3
    t = np.arange(N) % F
    H = np.tile(np.array([[2.0], [3.5], [5.0]]), (1, N))
    a = O.radius_variant(H, t, 0.7, 0.3, F, "shared", metric)
    b = O.radius_variant(H, t, 0.7, 0.3, F, "entropy", metric)
    assert np.allclose(a, b, rtol=1e-14, atol=0)


def test_entropy_disk_variant_is_the_pinned_radius():
    F, N = 4, 64
    t = np.arange(N) // 16
    H = np.linspace(1.0, 4.0, N)
    a = O.radius_variant(H[None, :], t, 0.3, 0.5, F, "entropy", "disk")[0]
    b = O.radius(H, t, 0.3, 0.5, F, N)
    assert np.array_equal(a, b)


def test_shared_budget_two_valued_closed_form_and_permutation_invariance():
    F, N, tau, gamma = 3, 120, 0.25, 0.4
    H = np.where(np.arange(N) % 2 == 0, 1.0, 4.0)[None, :]
    K = O.shared_budget_tokens(H, tau)
    assert abs(K[0] - tau * (math.e + math.e ** 4) / 2) < 1e-12
    # total budget of the head is unchanged: N * K_h = sum_i tau e^{H_i}
    assert abs(N * K[0] - tau * np.exp(H).sum()) < 1e-9
    t = np.arange(N) % F
    r = O.radius_variant(H, t, tau, gamma, F, "shared", "disk")
    rng = np.random.default_rng(0)
    r2 = O.radius_variant(H[:, rng.permutation(N)], t, tau, gamma, F, "shared", "disk")
    assert np.allclose(r, r2, rtol=1e-14, atol=0)   # only the summation order differs
    # queries of one frame share one radius; the radius holds K_h by equal area
    S = O.frame_energy(F, gamma)
    for f in range(F):
        rf = r[0, t == f]
        assert np.all(rf == rf[0])
        assert abs(math.pi * rf[0] ** 2 * S[f] - K[0]) < 1e-9 * K[0]


def test_line_mask_hand_example_wraps_across_rows():
    # W = 5: the query (x=4, y=1) has raster index n = 9; radius 2 keeps
    # n = 7..11 of its frame: (2,1), (3,1), (4,1), (0,2), (1,2)
    F, H, W = 1, 4, 5
    ck = O.token_coords(F, H, W)
    M = O.token_mask(np.array([2.0], np.float32), np.ones(1, np.float32),
                     np.array([[4, 1, 0]]), ck, "line", W)
    kept = sorted((int(x), int(y)) for x, y, _ in ck[M[0]])
    assert kept == [(0, 2), (1, 2), (2, 1), (3, 1), (4, 1)]


def test_line_mask_counts_are_interval_counts():
    F, H, W = 1, 15, 17
    ck = O.token_coords(F, H, W)
    cq = np.array([[8, 7, 0]])                         # n = 127, the frame holds 255 tokens
    for n2 in (0, 1, 2, 3, 4, 8, 9, 15, 16, 99, 100, 101, 5000):
        r = np.float32(math.sqrt(n2) + 1e-4)           # R2 in [n2, n2 + 1)
        M = O.token_mask(np.array([r]), np.ones(1, np.float32), cq, ck, "line", W)
        s = math.isqrt(n2)
        assert M.sum() == min(2 * s + 1, 127 + 1 + min(s, 127)), (n2, M.sum())


def test_line_budget_conservation():
    # every frame keeps 2*floor(R_t) + 1 keys (window inside the frame), so the
    # frames together hold K = 2 r L[t] tokens up to one key per frame
    F, H, W = 7, 64, 64
    gamma, tau = 0.3, 0.5
    N = F * H * W
    Hq = np.array([[math.log(N) - 2.0]])
    t_q = 3
    r = O.radius_variant(Hq, [t_q], tau, gamma, F, "entropy", "line")[0]
    K = tau * math.exp(Hq[0, 0])
    assert abs(2 * r[0] * O.frame_length(F, gamma)[t_q] - K) < 1e-9 * K
    phi32 = O.phi(np.arange(F), gamma).astype(np.float32)
    M = O.token_mask(r.astype(np.float32), phi32, np.array([[32, 32, t_q]]),
                     O.token_coords(F, H, W), "line", W)
    assert abs(M.sum() - K) <= F, (M.sum(), K)


def test_radial_bands_and_halving():
    d = np.arange(0, 1025)
    b = O.radial_band(d)
    assert b.tolist() == [math.floor(math.log2(x + 1)) for x in d]
    assert b[:16].tolist() == [0, 1, 1, 2, 2, 2, 2, 3, 3, 3, 3, 3, 3, 3, 3, 4]
    pd, pl = O.radial_phi(64, "disk"), O.radial_phi(64, "line")
    for dl in range(64):
        # area (disk) and length (line) halve once per band
        assert abs(pd[dl] ** 2 - 0.5 ** b[dl]) < 1e-15
        assert abs(pl[dl] - 0.5 ** b[dl]) < 1e-15


def test_radial_disk_support_grows_with_log_frames():
    # the query sits in frame 0; frames 2^b - 1 .. 2^(b+1) - 2 form band b and
    # each band holds about pi r0^2 keys, so F = 2^k - 1 frames give about
    # k pi r0^2 keys: support grows with log F (O(n log n) in total)
    H = W = 61
    r0 = np.float32(12.0)
    counts = []
    for k in (1, 2, 3, 4):
        F = 2 ** k - 1
        phi32 = O.radial_phi(F, "disk").astype(np.float32)
        M = O.token_mask(np.array([r0]), phi32, np.array([[30, 30, 0]]),
                         O.token_coords(F, H, W))
        counts.append(int(M.sum()))
    area = math.pi * float(r0) ** 2
    for k in range(1, 4):
        inc = counts[k] - counts[k - 1]
        assert abs(inc - area) < 0.1 * area, (k, inc, area)
    assert abs(counts[3] / counts[0] - 4.0) < 0.4


def test_radial_line_support_exact():
    # r0 = 64 and factors 2^-b are exact in fp32: band b has 2^b frames of
    # 2 * 64 * 2^-b + 1 keys, so F = 15 frames (bands 0..3) keep 4 * 128 + 15 keys
    F, H, W = 15, 21, 21
    phi32 = O.radial_phi(F, "line").astype(np.float32)
    M = O.token_mask(np.array([64.0], np.float32), phi32, np.array([[10, 10, 0]]),
                     O.token_coords(F, H, W), "line", W)
    assert int(M.sum()) == 4 * 128 + 15


def test_radial_single_frame_is_the_plain_disk():
    # one frame: phi_R(0) = 1 and the mask is the disk of radius r0 (the lattice
    # counts of the entropy-budget pins)
    ck = O.token_coords(1, 21, 21)
    for r0, count in ((1.0, 5), (2.0, 13), (3.0, 29)):
        M = O.token_mask(np.array([r0], np.float32), O.radial_phi(1).astype(np.float32),
                         np.array([[10, 10, 0]]), ck)
        assert int(M.sum()) == count


def _tiny_line(seed):
    F, H, W = 4, 8, 8
    pi = O.tile_major_order(F, H, W, (1, 4, 4))
    c = O.token_coords(F, H, W)[pi]
    rng = np.random.default_rng(seed)
    r = rng.uniform(0.0, 12.0, size=F * H * W).astype(np.float32)
    phi32 = O.phi(np.arange(F), 0.5).astype(np.float32)
    return c, r, phi32, W


def test_line_block_votes_brute_force_and_superset():
    c, r, phi32, W = _tiny_line(3)
    M = O.token_mask(r, phi32, c, c, "line", W)
    votes = O.block_votes(M, 16, 16)
    for qb in (0, 6, 15):
        for kb in (0, 9, 15):
            n = 0
            for i in range(qb * 16, qb * 16 + 16):
                for j in range(kb * 16, kb * 16 + 16):
                    dn = (c[i, 1] * W + c[i, 0]) - (c[j, 1] * W + c[j, 0])
                    R = np.float32(r[i] * phi32[abs(c[i, 2] - c[j, 2])])
                    n += int(dn * dn <= float(np.float32(R * R)))
            assert votes[qb, kb] == n
    bm = O.block_mask(r, phi32, c, 16, 16, 1, metric="line", W=W)
    qi, kj = np.nonzero(M)
    assert bm[qi // 16, kj // 16].all()
    assert np.array_equal(bm, votes >= 1)
