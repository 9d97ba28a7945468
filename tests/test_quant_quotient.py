"""The quantizer kernels' quotient x / s (Divisor in csrc/quantize.cu), emulated
step by step in IEEE fp32 on the CPU and checked against the oracle's codes.

The kernels replace the IEEE division per element with Markstein's
FMA-corrected quotient (P. Markstein, IBM J. Res. Dev. 34(1), 1990):
r = RN(1/s) once per scale, then q0 = RN(x r), e = RN(x - q0 s) (one FMA,
so x - q0 s is exact before its one rounding) and q = RN(q0 + e r) (one FMA).
Below the scale guard s < 2^-60 they divide. The oracle's codes are
RN(x / s) with one IEEE division (oracle/quant.py), so the two must agree on
every code.

Emulation: r, q0 are numpy fp32 operations (IEEE round to nearest even);
q0 * s and e * r are exact in float64 (24 x 24 bits), x - q0 s is exact in
float64 (its bits span 26 binades at most), so one cast to fp32 is the FMA's
single rounding. q0 + e r may round in float64; the float32 result can then
differ from the FMA's only when the float64 sum lies exactly on a float32
midpoint, and those sums are redone in rationals.

Scope: every BF16 x with |x| <= amax, both signs and -0 (whose E4M3 code
0x80 the correction step alone would lose), for each scale s = RN(amax / R),
R = 127 (INT8) and 448 (E4M3).
The default run takes every 13th positive BF16 amax plus the scales next to
the guard and at both ends of the range; FMHA_EXHAUSTIVE=1 takes all 32,639
(5.3e8 pairs per R, several minutes). Shifted inputs (x - mean, general fp32)
are sampled at random."""

import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import quant as oq

GUARD = np.float32(2.0 ** -60)
RANGES = {"int8": 127, "e4m3": 448}


def bf16_nonneg():
    """Every non-negative finite BF16 value, ascending, as float32."""
    return (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)


def bf16_within(xs, amax):
    """Every finite BF16 x with |x| <= amax, both signs (-0 included)."""
    a = xs[xs <= amax]
    return np.concatenate([a, -a])


def rn32_exact_sum(a64, b64):
    """RN32(a + b) for float64 a, b whose exact sum may need more than 53 bits."""
    t = a64 + b64
    f = t.astype(np.float32)
    lo = f.astype(np.float64)
    other = np.where(lo < t, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf)))
    on_midpoint = t == (lo + other.astype(np.float64)) / 2
    for j in np.nonzero(on_midpoint)[0]:
        exact = Fraction(float(a64[j])) + Fraction(float(b64[j]))
        c = np.float32(float(exact))
        cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
        f[j] = min(cands, key=lambda v: (abs(Fraction(float(v)) - exact), int(np.float32(v).view(np.uint32)) & 1))
    return f


def kernel_quotient(x, s, guard=True):
    """The kernel's x / s for fp32 arrays x and one fp32 scale s."""
    x = np.asarray(x, dtype=np.float32)
    s = np.float32(s)
    if guard and s < GUARD:
        return (x / s).astype(np.float32)
    with np.errstate(all="ignore"):
        r = np.float32(np.float32(1.0) / s)
        q0 = (x * r).astype(np.float32)
        e = (x.astype(np.float64) - q0.astype(np.float64) * np.float64(s)).astype(np.float32)
        q = rn32_exact_sum(q0.astype(np.float64), e.astype(np.float64) * np.float64(r))
        return np.copysign(q, x)  # the kernel restores the sign of x (of a zero quotient)


def codes_of(q, dtype):
    """Codes of fp32 quotients, encoded as the oracle encodes RN(x / s)."""
    return oq.codes_with_scale(q, np.float32(1.0), dtype)


def amax_sample(xs):
    amaxs = xs[1:]
    if os.environ.get("FMHA_EXHAUSTIVE") == "1":
        return amaxs
    pick = set(range(0, amaxs.size, 13)) | set(range(10)) | set(range(amaxs.size - 10, amaxs.size))
    # the scales on both sides of the guard, for both ranges
    for R in RANGES.values():
        k = int(np.searchsorted(amaxs, np.float32(GUARD * np.float32(R))))
        pick |= set(range(max(0, k - 5), min(amaxs.size, k + 5)))
    return amaxs[sorted(pick)]


@pytest.mark.parametrize("dtype", ["int8", "e4m3"])
def test_bf16_codes_match_ieee_division(dtype):
    R = np.float32(RANGES[dtype])
    xs = bf16_nonneg()
    checked = 0
    for amax in amax_sample(xs):
        s = oq.scale_from_amax(amax, dtype)
        x = bf16_within(xs, amax)
        got = codes_of(kernel_quotient(x, s), dtype)
        want = oq.codes_with_scale(x, s, dtype)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (f"amax {amax!r} s {s!r}: x {x[bad[0]]!r} code {got[bad[0]]} "
                               f"vs {want[bad[0]]}")
        checked += x.size
    assert checked > 10_000_000 and R > 0


@pytest.mark.parametrize("dtype", ["int8", "e4m3"])
def test_guard_is_needed_below_it(dtype):
    """Without the guard, the reciprocal of the smallest scales overflows and the
    quotient is NaN: the guard (not luck) keeps those codes right."""
    xs = bf16_nonneg()
    amax = xs[7]  # a subnormal BF16 amax: s ~ 1e-42, 1/s overflows
    s = oq.scale_from_amax(amax, dtype)
    assert s < GUARD
    x = bf16_within(xs, amax)
    assert np.isnan(kernel_quotient(x, s, guard=False)).any()
    assert np.array_equal(codes_of(kernel_quotient(x, s), dtype), oq.codes_with_scale(x, s, dtype))


@pytest.mark.parametrize("dtype", ["int8", "e4m3"])
def test_shifted_inputs_sampled(dtype):
    """General fp32 x (K smoothing subtracts a token mean): random x and scales
    s >= 2^-60, including quotients near every code's rounding boundary."""
    rng = np.random.default_rng(20261203)
    R = RANGES[dtype]
    for _ in range(40):
        log_s = rng.uniform(-60.0, 60.0)
        s = np.float32(2.0 ** log_s) * np.float32(rng.uniform(1.0, 2.0))
        s = max(s, GUARD)
        n = 50_000
        q_target = rng.uniform(-R, R, size=n)
        if dtype == "int8":  # near the half-integers where INT8 rounding flips
            q_target[: n // 2] = np.round(q_target[: n // 2]) + 0.5 + rng.uniform(-1e-5, 1e-5, size=n // 2)
        x = (q_target * np.float64(s)).astype(np.float32)
        got = codes_of(kernel_quotient(x, s), dtype)
        want = oq.codes_with_scale(x, s, dtype)
        assert np.array_equal(got, want), f"s {s!r}"


@pytest.mark.parametrize("dtype", ["int8", "e4m3"])
def test_uncorrected_quotient_would_fail(dtype):
    """The FMA correction is needed: RN(x * RN(1/s)) alone gives wrong codes
    within the same sample (so the sweep above can see a missing step)."""
    xs = bf16_nonneg()
    for amax in amax_sample(xs):
        s = oq.scale_from_amax(amax, dtype)
        if s < GUARD:
            continue
        x = bf16_within(xs, amax)
        q0 = (x * np.float32(np.float32(1.0) / s)).astype(np.float32)
        if not np.array_equal(codes_of(q0, dtype), oq.codes_with_scale(x, s, dtype)):
            return
    pytest.fail("no sampled scale distinguishes the uncorrected quotient")


def test_negative_zero_keeps_its_sign():
    """-0 / s is -0: E4M3 code 0x80, as the oracle encodes it."""
    q = kernel_quotient(np.array([-0.0, 0.0], dtype=np.float32), np.float32(0.01))
    assert np.signbit(q[0]) and not np.signbit(q[1])
    assert list(codes_of(q, "e4m3")) == [0x80, 0x00]


def test_nvfp4_block_quotients_match_division():
    """The exact NVFP4 path divides each 16-element block by e = decode(sb) * s_t
    with the same corrected quotient: its E2M1 codes equal those of RN(x / e)
    (oracle/nvfp4.py), on N(0,1) rows with outliers, values placed on and next
    to every E2M1 rounding boundary, and rows small enough that e falls below
    the guard."""
    from oracle import e4m3
    from oracle import nvfp4 as on

    rng = np.random.default_rng(4242)
    rows = [rng.standard_normal(4096).astype(np.float32) * np.where(rng.random(4096) < 0.01, 40.0, 1.0)]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float64)
    bound = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 10)])
    for scale in (1.0, 3.0e-3, 7.0e5, 2.0 ** -70):
        r = np.resize(np.concatenate([bound, -bound, [6.0, -6.0, 0.0, -0.0]]), 4096) * scale
        rows.append(r.astype(np.float32))
    x = np.stack(rows).astype(np.float32)
    x = x.view(np.uint32) & np.uint32(0xFFFF0000)  # exact BF16 values
    x = x.view(np.float32)
    _, sb_codes, st = on.quantize_per_token(x)
    checked = below = 0
    for i in range(x.shape[0]):
        for j in range(x.shape[1] // 16):
            e = np.float32(np.float32(e4m3.decode(np.array([sb_codes[i, j]]))[0]) * st[i])
            if e == 0:
                continue
            blk = x[i, 16 * j:16 * (j + 1)]
            got = on.e2m1_encode(kernel_quotient(blk, e))
            want = on.e2m1_encode((blk / e).astype(np.float32))
            assert np.array_equal(got, want), (i, j, e)
            checked += blk.size
            below += int(e < GUARD)
    assert checked > 20000 and below > 0


def test_int8_code_from_the_low_byte_of_a_shifted_sum():
    """The INT8 kernels read rint(q) from the low byte of RN(q + 1.5 * 2^23):
    in [2^23, 2^24) the float32 step is 1, so the addition rounds q to an integer
    (ties to even) and the low mantissa byte holds it in two's complement. Checked
    on every half-integer in [-127.5, 127.5], its float32 neighbours, and a dense
    sample of float32 values in that range; |q| <= 127 always holds there (s is
    amax / 127 rounded to nearest, so |x| / s exceeds 127 by at most a few ulps)."""
    halves = np.arange(-255, 256, dtype=np.float64) / 2.0
    h32 = halves.astype(np.float32)
    q = np.concatenate([h32, np.nextafter(h32, np.float32(-np.inf)), np.nextafter(h32, np.float32(np.inf)),
                        np.random.default_rng(9).uniform(-127.5, 127.5, 2_000_000).astype(np.float32)])
    q = q[np.abs(q) <= 127.5]
    shifted = (q + np.float32(1.5 * 2 ** 23)).astype(np.float32)
    low = (shifted.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8)
    want = np.rint(q).astype(np.int64)
    keep = np.abs(want) <= 127  # the 128s only arise beyond the range the kernels reach
    assert np.array_equal(low[keep].astype(np.int64), want[keep])
