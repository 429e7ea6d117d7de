"""The prefill kernel's FMA-pipe exponential (exp2_fma2 in pa_prefill.cu),
checked on the CPU against 2^z in float64.

The kernel computes part of its softmax weights as 2^z = 2^j * 2^f with j =
round(z) taken from z + 1.5 * 2^23, f in [-1/2, 1/2] and 2^f from a cubic;
the weights are then rounded to bf16 / fp16 (relative half-ulp 2^-9 / 2^-11).
This reads the four coefficients from the source and replays every step in
float32 (numpy), so a wrong coefficient, a wrong shifter or an exponent that
wraps fails here."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "paged_kv_cache_426_b200", "csrc", "pa_prefill.cu")


def coefficients():
    src = open(SRC).read()
    c = {int(k): np.float32(float(v)) for k, v in re.findall(r"kExpC(\d) = ([0-9.e+-]+)f", src)}
    assert sorted(c) == [0, 1, 2, 3]
    return c


def exp2_fma(z):
    """The kernel's steps, in float32."""
    c = coefficients()
    f32 = np.float32
    z = np.maximum(z.astype(f32), f32(-126.0))
    sh = f32(12582912.0)
    t = (z + sh).astype(f32)
    f = (z - (t - sh).astype(f32)).astype(f32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p.astype(np.float64) * f + c[k]).astype(f32)   # one fused step, rounded once
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(f32)


def test_relative_error_on_the_softmax_range():
    z = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    e = exp2_fma(z).astype(np.float64)
    rel = np.abs(e / np.exp2(z.astype(np.float64)) - 1)
    assert rel.max() < 1e-4                  # << 2^-11, the fp16 half-ulp of P
    # integers (f = 0) and half-integers (the ends of the reduced range)
    for zz in (0.0, 1.0, -1.0, 8.0, -60.0, 0.5, -0.5, 7.5):
        v = float(exp2_fma(np.array([zz]))[0])
        assert abs(v / 2.0 ** zz - 1) < 1e-4, zz


def test_far_below_the_range_is_tiny_and_non_negative():
    z = np.concatenate([np.linspace(-400.0, -125.0, 100001), [-np.inf]]).astype(np.float32)
    e = exp2_fma(z)
    assert np.all(np.isfinite(e)) and np.all(e >= 0) and np.all(e < 2.0 ** -124)
