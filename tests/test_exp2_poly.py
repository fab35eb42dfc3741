"""Error bound of the FMA-pipe 2^x used by the two-warpgroup attention kernel
for one score pair in four (Cody-Waite reduction + degree-3 minimax
polynomial).  The constants are read from the kernel source and the routine
is replayed in float32 arithmetic (each fused multiply-add rounded once);
the reference is numpy's exp2 in float64."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "entropy_adaptive_radius_b200", "csrc", "attention.cu")


def kernel_constants():
    text = open(SRC).read()
    body = text[text.index("float2 exp2_fma2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"make_float2\(([-0-9.e]+)f,", body)]
    # order in the source: magic, -magic, -1, c3, c2, c1, c0
    return nums


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_fma_model(x):
    magic, nmagic, neg1, c3, c2, c1, c0 = [np.float32(v) for v in kernel_constants()]
    x = np.maximum(np.float32(x), np.float32(-125.0)).astype(np.float32)
    t = (x + magic).astype(np.float32)
    n = (t + nmagic).astype(np.float32)
    f = fma32(n, neg1, x)
    q = fma32(f, c3, c2)
    q = fma32(q, f, c1)
    q = fma32(q, f, c0)
    bits = (t.view(np.int32).astype(np.int64) << 23) + q.view(np.int32).astype(np.int64)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32)


def test_constants_are_the_fitted_polynomial():
    magic, nmagic, neg1, c3, c2, c1, c0 = kernel_constants()
    assert magic == 12582912.0 and nmagic == -12582912.0 and neg1 == -1.0
    f = np.linspace(-0.5, 0.5, 100001)
    p = ((c3 * f + c2) * f + c1) * f + c0
    assert np.max(np.abs(p / np.exp2(f) - 1)) < 8e-5


def test_exp2_fma_relative_error_over_kernel_range():
    # the kernel evaluates 2^x for x = s*scale*log2(e) - m, x in (-inf, 8]
    x = np.concatenate([np.linspace(-124.0, 8.0, 2000001), np.linspace(-1.0, 1.0, 200001)])
    x = x.astype(np.float32)
    got = exp2_fma_model(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1e-4, rel.max()


def test_exp2_fma_tiny_and_special():
    # below the clamp the result is tiny (< 2^-124), never NaN or negative
    x = np.array([-125.0, -200.0, -1e30, 0.0, 8.0], np.float32)
    got = exp2_fma_model(x)
    assert np.all(np.isfinite(got)) and np.all(got >= 0)
    assert got[0] < 2.0 ** -124 and got[1] < 2.0 ** -124 and got[2] < 2.0 ** -124
    assert abs(got[3] - 1) < 1e-4 and abs(got[4] / 256 - 1) < 1e-4
