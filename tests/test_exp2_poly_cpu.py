"""Error bound of the prefill softmax's FMA-pipe exponential (`exp2_poly` in
csrc/attn_prefill_tc.cuh), evaluated step for step in float32 on the CPU.

The kernel computes a quarter of its 2^x with a degree-3 polynomial instead of
the MUFU unit.  P is rounded to bf16 afterwards, so the approximation must stay
well below half a bf16 ulp (2^-9 relative): the bound checked here is 1e-4.
The coefficients are read from the kernel source, so this checks the code that
runs, not a copy of it.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mla_latent_kv_47_b200", "csrc", "attn_prefill_tc.cuh")


def _coefficients():
    src = open(SRC).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("}")]
    m = re.search(r"fmaf\(fmaf\(fmaf\(([0-9.eE+-]+)f, f, ([0-9.eE+-]+)f\), f, ([0-9.eE+-]+)f\), f, ([0-9.eE+-]+)f\)", body)
    assert m, "exp2_poly's polynomial not found"
    c3, c2, c1, c0 = (np.float32(float(v)) for v in m.groups())
    assert "12582912.f" in body and "-126.f" in body
    return c0, c1, c2, c3


def exp2_poly_f32(x):
    """The kernel's steps in float32: clamp, round by the 1.5 * 2^23 constant,
    Horner with fused multiply-adds (emulated in float64, then rounded), and the
    exponent-field add."""
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    f = (x - (t - big).astype(np.float32)).astype(np.float32)
    fma = lambda a, b, c: (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)
    p = fma(fma(fma(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_below_a_bf16_half_ulp():
    # results from 2^-125 up (below it the exponent-field add reaches the
    # denormal range; such weights are nothing next to the row max of 1)
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    y = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_integers_and_halves():
    # at integers the polynomial's constant term alone is used; at +-1/2 the
    # ends of the fitted interval
    for x in (-3.0, 0.0, 1.0, 7.0, -0.5, 0.5, -2.5, 3.5):
        y = float(exp2_poly_f32(np.float32(x)))
        assert abs(y / 2.0 ** x - 1) < 1e-4, (x, y)


def test_masked_keys_give_a_negligible_weight():
    # masked (future) keys enter as -inf: the clamp makes them 2^-126, which
    # is nonnegative and below any weight that can matter next to the row max (1)
    y = float(exp2_poly_f32(np.float32(-np.inf)))
    assert 0.0 <= y <= 2.0 ** -125
