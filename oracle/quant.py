"""Block quantization: amax -> scale -> INT8 / E4M3 codes, in exact IEEE float32.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix: Q/K/V may each be Int8, BF16 or E4M3, and SageAttention
scales them block by block rather than per tensor, because block-wise scaling
keeps more precision on outlier-heavy attention maps ("FlashInfer DiT
optimization: SageAttention and Int8/FP8 mixed-precision kernels", intro,
section 2 and "Why" item 2). The per-block recipe amax -> scale -> code and the
granularities (per 128-token Q block, per 64-token K block, per channel, per
head, per tensor) come from the workload definitions this library is built
for. The pages are silent on everything below; the readings taken are:

* amax = max |x| over the block, x exact in float32 (BF16 inputs convert
  exactly).
* scale = float32(amax) / float32(R), one IEEE round-to-nearest-even division,
  R = 127 for INT8 and 448 for E4M3. The stored scale is this dequantization
  multiplier (x ~= code * scale), not its reciprocal.
* amax = 0 gives scale = 1.0 and all-zero codes.
* code = float32(x) / scale, one IEEE division per element, then
  INT8: round half to even, clamp to [-127, 127] (symmetric range);
  E4M3: round to nearest even with saturation to +-448 (``e4m3.encode``).
* A ragged last token block covers the remaining rows.
* Granularities ("kind") and scale layouts, for x of shape [B, S, H, D]:
    per_tensor       scales [1]            one over everything
    per_head         scales [B, H]         one per (b, h) over S x D
    per_token_block  scales [B, H, nblk]   one per (b, h, rows_per_block tokens) over rows x D
    per_channel      scales [B, H, D]      one per (b, h, d) over all S tokens
"""

import numpy as np

from . import e4m3

RANGE = {"int8": 127.0, "e4m3": 448.0}
KINDS = ("per_tensor", "per_head", "per_token_block", "per_channel")


def scale_from_amax(amax_f32, out_dtype):
    """scale = fp32(amax) / fp32(R), 1.0 where amax == 0."""
    amax_f32 = np.asarray(amax_f32, dtype=np.float32)
    r = np.float32(RANGE[out_dtype])
    scale = (amax_f32 / r).astype(np.float32)  # numpy float32 division is IEEE RN-even
    return np.where(amax_f32 == 0, np.float32(1.0), scale).astype(np.float32)


def codes_with_scale(x_f32, scale_f32, out_dtype):
    """Codes of x for a given (broadcastable) scale: RN(fp32(x) / scale)."""
    q = (np.asarray(x_f32, dtype=np.float32) / np.asarray(scale_f32, dtype=np.float32)).astype(np.float32)
    if out_dtype == "int8":
        return np.clip(np.rint(q), -127, 127).astype(np.int8)
    if out_dtype == "e4m3":
        return e4m3.encode(q)
    raise ValueError(out_dtype)


def num_blocks(S, rows_per_block):
    return (S + rows_per_block - 1) // rows_per_block


def channel_mean(x):
    """Token mean of x [B, S, H, D] for every (b, h, d) -> float32 [B, H, D].

    K smoothing. SageAttention quantizes K after subtracting K's mean over the
    tokens (Zhang et al., "SageAttention: Accurate 8-Bit Attention for
    Plug-and-play Inference Acceleration", 2024, smoothing of K). The pages
    name SageAttention and its block-wise scale factors, but not this step.
    The readings taken are:
    * the mean runs over all S tokens of one (b, h), separately per channel d;
    * the S values (exact in float32) are summed in float64, the sum is
      divided by S in float64, and the quotient is rounded once to float32;
    * S = 0 gives a zero mean.
    A shift that is constant over the tokens of one (b, h) moves every score of
    a query row by the same amount, q . mean. Softmax ignores that, so O is
    unchanged, and the log-sum-exp moves by softmax_scale * q . mean.
    """
    x = np.asarray(x, dtype=np.float32)
    B, S, H, D = x.shape
    if S == 0:
        return np.zeros((B, H, D), dtype=np.float32)
    total = x.astype(np.float64).sum(axis=1)  # [B, H, D]
    return (total / np.float64(S)).astype(np.float32)


def quantize_blockwise(x, out_dtype, kind, rows_per_block=None, shift=None):
    """x: float32 array [B, S, H, D] (exact BF16 values). Returns (codes, scales).

    codes has x's shape (int8, or uint8 E4M3 bit patterns); scales is float32
    with the layout of ``kind`` given in the module docstring.

    shift (optional, float32 [B, H, D], e.g. ``channel_mean(x)``): the values
    quantized are x - shift, one float32 round-to-nearest-even subtraction per
    element, and every block's amax is taken over those differences. The codes
    then dequantize to x - shift.
    """
    x = np.asarray(x, dtype=np.float32)
    B, S, H, D = x.shape
    if shift is not None:
        sh = np.asarray(shift, dtype=np.float32)
        if sh.shape != (B, H, D):
            raise ValueError(f"shift must have shape {(B, H, D)}, got {sh.shape}")
        x = (x - sh[:, None, :, :]).astype(np.float32)
    codes = np.zeros(x.shape, dtype=np.int8 if out_dtype == "int8" else np.uint8)
    if kind == "per_tensor":
        scale = scale_from_amax(np.max(np.abs(x)) if x.size else np.float32(0), out_dtype)
        codes[...] = codes_with_scale(x, scale, out_dtype)
        return codes, np.array([scale], dtype=np.float32)
    if kind == "per_head":
        scales = np.zeros((B, H), dtype=np.float32)
        for b in range(B):
            for h in range(H):
                blk = x[b, :, h, :]
                s = scale_from_amax(np.max(np.abs(blk)) if blk.size else np.float32(0), out_dtype)
                scales[b, h] = s
                codes[b, :, h, :] = codes_with_scale(blk, s, out_dtype)
        return codes, scales
    if kind == "per_token_block":
        if not rows_per_block or rows_per_block <= 0:
            raise ValueError("per_token_block needs rows_per_block > 0")
        nblk = num_blocks(S, rows_per_block)
        scales = np.zeros((B, H, nblk), dtype=np.float32)
        for b in range(B):
            for h in range(H):
                for i in range(nblk):
                    s0, s1 = i * rows_per_block, min(S, (i + 1) * rows_per_block)
                    blk = x[b, s0:s1, h, :]
                    s = scale_from_amax(np.max(np.abs(blk)), out_dtype)
                    scales[b, h, i] = s
                    codes[b, s0:s1, h, :] = codes_with_scale(blk, s, out_dtype)
        return codes, scales
    if kind == "per_channel":
        scales = np.zeros((B, H, D), dtype=np.float32)
        for b in range(B):
            for h in range(H):
                for d in range(D):
                    col = x[b, :, h, d]
                    s = scale_from_amax(np.max(np.abs(col)) if col.size else np.float32(0), out_dtype)
                    scales[b, h, d] = s
                    codes[b, :, h, d] = codes_with_scale(col, s, out_dtype)
        return codes, scales
    raise ValueError(kind)


def dequantize(codes, scales, out_dtype, kind, rows_per_block=None):
    """codes, scales as returned by ``quantize_blockwise`` -> float64 [B, S, H, D].

    code * scale is exact in float64 (an 8-bit integer or E4M3 value times a
    float32).
    """
    if out_dtype == "int8":
        vals = np.asarray(codes, dtype=np.int8).astype(np.float64)
    else:
        vals = e4m3.decode(codes)
    B, S, H, D = vals.shape
    sc = np.asarray(scales, dtype=np.float32).astype(np.float64)
    if kind == "per_tensor":
        return vals * sc.reshape(())
    if kind == "per_head":
        return vals * sc[:, None, :, None]
    if kind == "per_token_block":
        idx = np.arange(S) // rows_per_block
        per_row = sc[:, :, idx]  # [B, H, S]
        return vals * per_row.transpose(0, 2, 1)[:, :, :, None]
    if kind == "per_channel":
        return vals * sc[:, None, :, :]
    raise ValueError(kind)
