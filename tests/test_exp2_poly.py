"""The FMA-pipe exp2 of the attention kernel (exp2_poly_x2 in attn_kernel.cuh),
emulated step by step in IEEE fp32 on the CPU and checked against 2^x.

The kernel computes a share of the softmax exponentials without MUFU: x is
clamped to [-125, inf), n = rint(x) by adding 1.5 * 2^23, f = x - n in
[-1/2, 1/2], 2^f by a polynomial in f (Horner, fused multiply-adds), and 2^n
is added to the exponent field as the integer n << 23. The coefficients are
read from the kernel source, so the bound tested here is the one the kernel
runs with. Rounding of each fp32 operation is emulated exactly (an fp32
product is exact in fp64, and fma(a, b, c) is rounded once from the exact
value computed with Python fractions where float64 would round twice).
"""

import os
import re
from fractions import Fraction

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "precision_attention_fmha_b200", "csrc", "attn_kernel.cuh")
MAGIC = np.float32(12582912.0)


def coefficients():
    s = open(SRC).read()
    body = s[s.index("__device__ __forceinline__ void exp2_poly_x2"):]
    body = body[:body.index("\n}\n")]
    deg3 = body[body.index("DEG == 3"):body.index("} else {")]
    deg2 = body[body.index("} else {"):]
    num = r"([0-9.]+)f"
    c3 = [float(v) for v in re.findall(num, deg3)]
    c2 = [float(v) for v in re.findall(num, deg2)]
    # ffma2 operand order: (f * a + b), then (p * f + c), ... -> Horner from the top
    return {3: [np.float32(c3[0]), np.float32(c3[2]), np.float32(c3[4]), np.float32(c3[6])],
            2: [np.float32(c2[0]), np.float32(c2[2]), np.float32(c2[4])]}


def fma32(a, b, c):
    """fp32 fused multiply-add, rounded once (exact rational then one rounding)."""
    exact = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    lo = np.float32(float(exact))
    # float(exact) rounds to float64 first; fix the rare double-rounding case by
    # picking the fp32 neighbour nearest to the exact value (ties to even).
    cands = [np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))]
    best = min(cands, key=lambda v: (abs(Fraction(float(v)) - exact), int(np.float32(v).view(np.uint32)) & 1))
    return np.float32(best)


def exp2_poly(x, deg, coef):
    x = np.float32(max(np.float32(x), np.float32(-125.0)))
    j = np.float32(x + MAGIC)
    n = np.float32(j - MAGIC)
    f = np.float32(x - n)
    c = coef[deg]
    p = fma32(f, c[0], c[1])
    for ci in c[2:]:
        p = fma32(p, f, ci)
    bits = (int(p.view(np.uint32)) + ((int(j.view(np.uint32)) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    return np.uint32(bits).view(np.float32)


@pytest.mark.parametrize("deg,bound", [(2, 1.8e-3), (3, 8e-5)])
def test_relative_error_bound(deg, bound):
    coef = coefficients()
    rng = np.random.default_rng(7)
    xs = np.concatenate([np.linspace(-124.0, 9.5, 1501), rng.uniform(-30.0, 9.0, 1500),
                         np.arange(-120, 10) + 0.5, np.arange(-120, 10).astype(np.float64)]).astype(np.float32)
    worst = 0.0
    for x in xs:
        got = float(exp2_poly(x, deg, coef))
        ref = 2.0 ** float(x)
        worst = max(worst, abs(got - ref) / ref)
    assert worst <= bound, (deg, worst)


@pytest.mark.parametrize("deg", [2, 3])
def test_hidden_scores_and_clamp_give_a_tiny_normal_value(deg):
    coef = coefficients()
    for x in (-np.inf, np.float32(-1e30), np.float32(-126.0), np.float32(-125.0)):
        v = exp2_poly(np.float32(x), deg, coef)
        assert np.isfinite(v) and 0.0 < float(v) < 2.0 ** -123, (x, v)


def test_integer_arguments_are_powers_of_two_within_the_bound():
    coef = coefficients()
    for n in range(-120, 10):
        v = float(exp2_poly(np.float32(n), 2, coef))
        assert abs(v / 2.0 ** n - 1.0) <= 1.8e-3
