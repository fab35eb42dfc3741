"""Pins of the oracle's FP8 (E4M3) score path (CPU): the rounding against
the E4M3 format written out bit by bit, the per-block quantization against
its error bound, and FP8 attention against the pinned exact attention on
inputs that E4M3 represents exactly."""

import numpy as np

from oracle import tra_oracle as O


def e4m3_values():
    """Every finite E4M3 value from the bit-level definition: sign, 4-bit
    exponent e (bias 7), 3-bit mantissa m; e = 0 is subnormal (m/8 * 2^-6);
    code 0x7F (e = 15, m = 7) is NaN, so the largest finite is 1.75 * 2^8."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
            vals.append((v, m))
    return vals


def test_e4m3_representable_values_are_fixed_points():
    vals = e4m3_values()
    assert max(v for v, _ in vals) == 448.0
    assert len({v for v, _ in vals}) == 127          # +0 and 126 positive values
    x = np.array([v for v, _ in vals] + [-v for v, _ in vals])
    assert np.array_equal(O.round_e4m3(x), x)


def test_e4m3_rounds_to_nearest_even_and_saturates():
    vals = sorted(set(e4m3_values()))
    for (a, ma), (b, mb) in zip(vals, vals[1:]):
        mid = 0.5 * (a + b)
        even = a if ma % 2 == 0 else b
        assert O.round_e4m3(np.array([mid]))[0] == even, (a, b)
        assert O.round_e4m3(np.array([a + 0.25 * (b - a)]))[0] == a
        assert O.round_e4m3(np.array([b - 0.25 * (b - a)]))[0] == b
    assert O.round_e4m3(np.array([1e6, -600.0, 449.0]))[0] == 448.0
    assert np.array_equal(O.round_e4m3(np.array([-600.0, 449.0])), [-448.0, 448.0])


def test_quantize_blocks_scale_and_error_bound():
    rng = np.random.default_rng(1)
    X = rng.normal(size=(2, 300, 32)) * np.array([0.01, 3.0])[:, None, None]
    X[1, 128:256] = 0.0                               # an all-zero block
    codes, scales = O.quantize_e4m3_blocks(X, 128)
    assert scales.shape == (2, 3) and scales[1, 1] == np.float32(1.0)
    assert np.all(codes[1, 128:256] == 0.0)
    X32 = X.astype(np.float32).astype(np.float64)
    for h in range(2):
        for b in range(3):
            blk = X32[h, b * 128:(b + 1) * 128]
            c = codes[h, b * 128:(b + 1) * 128]
            if not blk.any():
                continue
            # the block's largest magnitude lands on +-448
            i = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
            assert abs(c[i]) == 448.0
            sc = float(scales[h, b])
            assert scales[h, b] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448.0))
            y = blk / sc
            # half an E4M3 ulp: 2^-4 relative in the normal range, 2^-10 absolute below
            bound = np.where(np.abs(y) >= 2.0 ** -6, np.abs(y) * 2.0 ** -4, 2.0 ** -10)
            assert np.all(np.abs(c - y) <= bound * (1 + 1e-6) + 1e-7 * np.abs(y))


def test_fp8_attention_equals_exact_attention_on_representable_inputs():
    # entries in {-1, -1/2, 0, 1/2, 1} with a +-1 in every block: scale = fl32(1/448)
    # and x / scale lands on 0, +-224 or +-448, all E4M3 values
    rng = np.random.default_rng(2)
    heads, N, d, B = 2, 200, 16, 64
    Q = rng.choice([-1.0, -0.5, 0.0, 0.5, 1.0], size=(heads, N, d))
    K = rng.choice([-1.0, -0.5, 0.0, 0.5, 1.0], size=(heads, N, d))
    Q[:, ::B, 0] = 1.0
    K[:, ::B, 0] = -1.0
    V = rng.normal(size=(heads, N, d))
    Q8, qs = O.quantize_e4m3_blocks(Q, B)
    K8, ks = O.quantize_e4m3_blocks(K, B)
    assert np.array_equal(Q8, Q * 448.0) and np.array_equal(K8, K * 448.0)
    nb = -(-N // B)
    mask = rng.random((heads, nb, nb)) < 0.5
    mask[:, np.arange(nb), np.arange(nb)] = True
    O8, L8 = O.sparse_attention_fp8qk(Q8, qs, K8, ks, V, mask, B, B, 0.25)
    Oe, Le = O.sparse_attention(Q, K, V, mask, B, B, 0.25)
    # only the fp32 rounding of 1/448 separates the two score scalings
    assert np.max(np.abs(O8 - Oe)) < 1e-5 and np.max(np.abs(L8 - Le)) < 1e-5
    # the row form agrees with the full form
    rows = np.array([0, 63, 64, 199])
    Or, Lr = O.sparse_attention_fp8qk(Q8, qs, K8, ks, V, mask, B, B, 0.25, rows=rows, head=1)
    assert np.allclose(Or, O8[1][rows], rtol=0, atol=1e-12)
    assert np.allclose(Lr, L8[1][rows], rtol=0, atol=1e-12)
