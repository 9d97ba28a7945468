"""OCP 8-bit floating point E4M3 ("E4M3FN") codec, from the format definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name the format only as "E4M3" ("FlashInfer DiT optimization:
SageAttention and Int8/FP8 mixed-precision kernels", section 3, and "FlashInfer
FP8/BF16 mixed-precision attention for Blackwell", introduction). The reading
taken here: the OCP FP8 E4M3 variant used by every Blackwell tensor core --
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
NaN = S.1111.111, largest finite magnitude 1.75 * 2^8 = 448, smallest normal
2^-6, subnormals k * 2^-9 for k = 1..7.

Encoding is round-to-nearest, ties to even, from the exact value of the input,
saturating to +-448 (the "satfinite" behaviour): the quantizer divides by
amax/448, so a value landing a rounding step above 448 must clamp, not turn
into NaN.
"""

import numpy as np

MAX = 448.0
MIN_NORMAL = 2.0 ** -6
SUBNORMAL_STEP = 2.0 ** -9  # quantum of the subnormal range (and of the first normal binade)


def decode(codes):
    """Codes (uint8 array) -> float64 values. NaN codes decode to NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp_field = (c >> 3) & 0xF
    mant = (c & 0x7).astype(np.float64)
    normal = (1.0 + mant / 8.0) * np.exp2(exp_field.astype(np.float64) - 7.0)
    subnormal = mant * SUBNORMAL_STEP
    val = np.where(exp_field == 0, subnormal, normal)
    val = np.where((exp_field == 0xF) & ((c & 0x7) == 0x7), np.nan, val)
    return sign * val


def encode(x):
    """Values (any float array, taken exactly in float64) -> uint8 codes.

    Round to nearest, ties to even; magnitudes beyond 448 saturate to 448.
    NaN encodes to 0x7F (sign kept).
    """
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    # Quantum of the binade that holds a: 2^(e-3) for a in [2^e, 2^(e+1)),
    # and the fixed subnormal step below 2^-6.
    _, e2 = np.frexp(np.where(a > 0, a, 1.0))  # a = f * 2^e2 with f in [0.5, 1)
    e = e2.astype(np.int64) - 1  # a in [2^e, 2^(e+1))
    e = np.maximum(e, -6)  # the subnormal range shares the 2^-6 binade's quantum
    quantum = np.exp2((e - 3).astype(np.float64))
    steps = np.rint(a / quantum)  # exact division by a power of two; rint ties to even
    r = steps * quantum
    r = np.minimum(r, MAX)
    # Bits from the rounded magnitude (which may have carried into the next binade).
    _, re2 = np.frexp(np.where(r > 0, r, 1.0))
    re = re2.astype(np.int64) - 1
    is_sub = r < MIN_NORMAL
    exp_field = np.where(is_sub, 0, re + 7)
    mant = np.where(is_sub, r / SUBNORMAL_STEP, (r / np.exp2(re.astype(np.float64)) - 1.0) * 8.0)
    mant = np.rint(mant).astype(np.int64)  # exact integers already
    code = (exp_field << 3) | mant
    code = np.where(nan, 0x7F, code)
    code = np.where(neg, code | 0x80, code)
    return code.astype(np.uint8)


def all_finite_codes():
    """The 254 finite codes (both signs), as uint8."""
    c = np.arange(256, dtype=np.uint8)
    return c[~np.isnan(decode(c))]
