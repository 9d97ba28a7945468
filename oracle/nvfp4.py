"""Per-token NVFP4 quantization, from the format definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The page ("FlashInfer per-token NVFP4 quantization kernel", introduction and
sections 1-2) names the operation -- NVFP4 codes with a per-token scale -- and
two properties of its kernel: the input row stays on chip between the pass
that finds its amax and the pass that quantizes it, and a "fast math" path
can be switched off. It states no formula. The readings taken here:

* Element format E2M1 (FP4): 1 sign bit, 2 exponent bits with bias 1, 1
  mantissa bit, no infinities or NaN. Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
  Encoding rounds to nearest, ties to the even mantissa bit, and saturates to
  +-6.
* Two-level scale (NVFP4): 16 consecutive elements of a row share one E4M3
  block scale; each token (row) has one fp32 scale s_t that maps the row's
  amax onto the largest block scale times the largest element, 448 * 6:
      s_t  = fp32(amax_row) / 2688              (1.0 when amax_row == 0)
      sb   = E4M3( (amax_blk / s_t) / 6 )       (two IEEE fp32 divisions; RN, satfinite)
      e    = fp32( decode(sb) * s_t )           (the block's element scale)
      code = E2M1( x / e )                      (IEEE fp32 division; all zero when e == 0)
  Fast math (the page's switch): code = E2M1( x * fp32(1 / e) ), one
  reciprocal per block instead of one division per element.
  Dequantization: x ~= e2m1(code) * decode(sb) * s_t.
* Layout: a row of K values (K % 16 == 0) gives K/2 bytes of codes, element 2i
  in the low nibble of byte i and element 2i+1 in the high nibble, K/16 E4M3
  block-scale bytes and one fp32 token scale.
"""

import numpy as np

from . import e4m3

E2M1_MAX = 6.0
ROW_RANGE = np.float32(448.0 * 6.0)  # 2688, exact in fp32
BLOCK = 16


def e2m1_decode(codes):
    """4-bit codes (0..15) -> float64 values."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    exp_field = (c >> 1) & 0x3
    mant = (c & 0x1).astype(np.float64)
    normal = (1.0 + mant / 2.0) * np.exp2(exp_field.astype(np.float64) - 1.0)
    subnormal = mant * 0.5
    return sign * np.where(exp_field == 0, subnormal, normal)


def e2m1_encode(x):
    """Values (taken exactly in float64) -> 4-bit codes: round to nearest,
    ties to the code with an even mantissa bit, saturate to +-6. The sign of
    zero is kept."""
    x = np.asarray(x, dtype=np.float64)
    mags = e2m1_decode(np.arange(8))  # 0, .5, 1, 1.5, 2, 3, 4, 6 (increasing)
    a = np.minimum(np.abs(x), E2M1_MAX)
    codes = np.zeros(x.shape, dtype=np.int64)
    # nearest by exhaustive comparison over the 8 magnitudes; ties -> even code
    best = np.full(x.shape, np.inf)
    for c in range(8):
        d = np.abs(a - mags[c])
        better = (d < best) | ((d == best) & (c % 2 == 0))
        codes = np.where(better, c, codes)
        best = np.where(better, d, best)
    neg = np.signbit(x)
    return (codes | np.where(neg, 8, 0)).astype(np.uint8)


def quantize_per_token(x, fast_math=False):
    """x: float32 array [rows, K] (exact BF16 values), K % 16 == 0.

    Returns (codes uint8 [rows, K/2], block_scales uint8 [rows, K/16] (E4M3),
    token_scales float32 [rows])."""
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    assert K % BLOCK == 0
    nb = K // BLOCK
    codes4 = np.zeros((rows, K), dtype=np.uint8)
    sb_codes = np.zeros((rows, nb), dtype=np.uint8)
    st = np.ones(rows, dtype=np.float32)
    for r in range(rows):
        amax = np.float32(np.max(np.abs(x[r]))) if K else np.float32(0)
        s_t = np.float32(1.0) if amax == 0 else np.float32(amax / ROW_RANGE)
        st[r] = s_t
        for j in range(nb):
            blk = x[r, j * BLOCK:(j + 1) * BLOCK]
            amax_b = np.float32(np.max(np.abs(blk)))
            q = np.float32(np.float32(amax_b / s_t) / np.float32(6.0))
            sb = e4m3.encode(np.array([q]))[0]
            sb_codes[r, j] = sb
            e = np.float32(np.float32(e4m3.decode(np.array([sb]))[0]) * s_t)
            if e == 0:
                codes4[r, j * BLOCK:(j + 1) * BLOCK] = 0
                continue
            if fast_math:
                y = (blk * np.float32(np.float32(1.0) / e)).astype(np.float32)
            else:
                y = (blk / e).astype(np.float32)
            codes4[r, j * BLOCK:(j + 1) * BLOCK] = e2m1_encode(y)
    packed = (codes4[:, 0::2] | (codes4[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb_codes, st


def dequantize(packed, block_scales, token_scales):
    """-> float64 [rows, K]."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    c = np.zeros((rows, 2 * half), dtype=np.uint8)
    c[:, 0::2] = packed & 0xF
    c[:, 1::2] = packed >> 4
    vals = e2m1_decode(c)
    sb = e4m3.decode(block_scales).astype(np.float64)
    per_elem = np.repeat(sb, BLOCK, axis=1) * np.asarray(token_scales, dtype=np.float32).astype(np.float64)[:, None]
    return vals * per_elem
