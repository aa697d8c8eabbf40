"""The prefill attention kernel computes a share of its softmax exponentials 2^x on the
FMA pipe: x = j + f with j the nearest integer (from a 1.5 * 2^23 shifter), 2^f by a cubic
on [-1/2, 1/2], 2^j added into the exponent field.  This replays those steps in float32
with the kernel's own coefficients and bounds the relative error against 2^x; the bf16
rounding that the probabilities then get is 2^-9 relative, so 1e-4 leaves it untouched."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "recurrent_depth_moe_b200", "csrc", "k_attn_tc.cu")


def _coefficients():
    text = open(SRC).read()
    c = {k: float(v) for k, v in re.findall(r"EXP2_(C[0-3]) = ([-0-9.e]+)f", text)}
    assert sorted(c) == ["C0", "C1", "C2", "C3"], c
    return [np.float32(c[f"C{i}"]) for i in range(4)]


def _fma(a, b, c):
    # one rounding, as the hardware FMA (the f32 product is exact in f64)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _poly_exp2(x):
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    jf = (t - shifter).astype(np.float32)
    f = _fma(jf, np.full_like(jf, -1.0), x)
    p = _fma(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma(p, f, np.full_like(f, c1))
    p = _fma(p, f, np.full_like(f, c0))
    return (p.view(np.int32) + (t.view(np.int32) << 23)).view(np.float32)


def test_relative_error_over_the_softmax_range():
    # the running max is raised lazily (by more than 2^8), so x reaches +8
    x = np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32)
    got = _poly_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1e-4


def test_reduction_at_half_integers_and_integers():
    # the nearest-integer split switches j at odd multiples of 1/2: both sides agree there
    k = np.arange(-60, 8, dtype=np.float32)
    for x in (k, k + np.float32(0.5), k - np.float32(0.5), np.nextafter(k + np.float32(0.5), np.float32(-200))):
        got = _poly_exp2(x).astype(np.float64)
        want = np.exp2(x.astype(np.float64))
        assert np.max(np.abs(got - want) / want) < 1e-4


def test_masked_scores_are_clamped_to_a_negligible_value():
    got = _poly_exp2(np.array([-np.inf, -1e30, -126.0], dtype=np.float32))
    assert np.all(got > 0) and np.all(got < 3e-38)
