"""Pins for the oracle's block quantizer (CPU only).

Pinned against closed forms and properties that a wrong block partition, a
wrong scale formula, a wrong rounding mode or a transposed scale layout
would break: hand-built ties, the max code of every block being exactly +-R,
the dequantization error bound, block independence, and agreement between
granularities that must coincide.
"""

import numpy as np
import pytest

from fractions import Fraction

from oracle import e4m3, quant


def _bf16_like(rng, shape, scale=1.0):
    import torch

    x = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32))
    return x.to(torch.bfloat16).to(torch.float32).numpy()


def test_int8_ties_round_half_even():
    # amax = 127 gives scale exactly 1.0, so codes are rint(x) directly.
    x = np.array([127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, -126.5], dtype=np.float32)
    codes, scales = quant.quantize_blockwise(x.reshape(1, -1, 1, 1), "int8", "per_tensor")
    assert scales[0] == np.float32(1.0)
    assert codes.ravel().tolist() == [127, 0, 2, 2, 0, -2, -2, 4, -126]


def test_int8_scale_is_amax_over_127_in_float32():
    # amax = 254 -> scale = 2 exactly; x = 3 -> 1.5 -> 2 (even); x = 5 -> 2.5 -> 2.
    x = np.array([254.0, 3.0, 5.0, -7.0], dtype=np.float32)
    codes, scales = quant.quantize_blockwise(x.reshape(1, -1, 1, 1), "int8", "per_tensor")
    assert scales[0] == np.float32(2.0)
    assert codes.ravel().tolist() == [127, 2, 2, -4]


def test_e4m3_unit_scale_equals_codec():
    rng = np.random.default_rng(1)
    x = _bf16_like(rng, (1, 64, 1, 32), 20.0)
    x[0, 0, 0, 0] = 448.0  # amax 448 -> scale 1
    x[0, 1, 0, 0] = -1.0
    codes, scales = quant.quantize_blockwise(x, "e4m3", "per_tensor")
    assert scales[0] == np.float32(1.0)
    assert np.array_equal(codes, e4m3.encode(x))


@pytest.mark.parametrize("out", ["int8", "e4m3"])
@pytest.mark.parametrize("kind,rpb", [("per_tensor", None), ("per_head", None),
                                      ("per_token_block", 64), ("per_token_block", 128),
                                      ("per_channel", None)])
def test_every_block_hits_full_range_and_error_bound(out, kind, rpb):
    rng = np.random.default_rng(2)
    B, S, H, D = 2, 200, 3, 16  # S=200: ragged last token block
    # give different blocks very different magnitudes so a wrong partition shows
    mag = np.exp2(rng.integers(-6, 6, size=(B, S, H, D))).astype(np.float32)
    x = _bf16_like(rng, (B, S, H, D)) * mag
    codes, scales = quant.quantize_blockwise(x, out, kind, rpb)
    xhat = quant.dequantize(codes, scales, out, kind, rpb)
    R = quant.RANGE[out]
    vals = codes.astype(np.float64) if out == "int8" else e4m3.decode(codes)
    # per-block max |code| is exactly R
    if kind == "per_tensor":
        groups = [np.abs(vals).max()]
    elif kind == "per_head":
        groups = [np.abs(vals[b, :, h, :]).max() for b in range(B) for h in range(H)]
    elif kind == "per_token_block":
        groups = [np.abs(vals[b, i:i + rpb, h, :]).max() for b in range(B) for h in range(H)
                  for i in range(0, S, rpb)]
    else:
        groups = [np.abs(vals[b, :, h, d]).max() for b in range(B) for h in range(H) for d in range(D)]
    assert all(g == R for g in groups)
    # error bound: INT8 |x - xhat| <= scale/2 (+ float32 division slop);
    # E4M3: half a quantum of the value's binade (relative 2^-4), or 2^-10*scale below 2^-6.
    scale_full = quant.dequantize(np.ones_like(codes) if out == "int8" else
                                  np.full_like(codes, 0x38), scales, out, kind, rpb)
    err = np.abs(x.astype(np.float64) - xhat)
    if out == "int8":
        assert np.all(err <= scale_full * (0.5 + 1e-5))
    else:
        bound = np.maximum(np.abs(x) * 2.0 ** -4, scale_full * 2.0 ** -10) * (1 + 1e-5)
        assert np.all(err <= bound)


def test_zero_block_gets_unit_scale_and_zero_codes():
    x = np.zeros((1, 130, 2, 8), dtype=np.float32)
    x[0, :128, 1, :] = 3.0
    codes, scales = quant.quantize_blockwise(x, "int8", "per_token_block", 128)
    assert scales[0, 0, 0] == 1.0 and scales[0, 0, 1] == 1.0 and scales[0, 1, 1] == 1.0
    assert scales[0, 1, 0] == np.float32(np.float32(3.0) / np.float32(127.0))
    assert np.all(codes[0, :, 0, :] == 0)


def test_block_independence():
    rng = np.random.default_rng(3)
    x = _bf16_like(rng, (1, 256, 2, 16))
    c0, s0 = quant.quantize_blockwise(x, "int8", "per_token_block", 64)
    y = x.copy()
    y[0, 70, 1, 5] = 1000.0  # lands in token block 1 of head 1
    c1, s1 = quant.quantize_blockwise(y, "int8", "per_token_block", 64)
    changed = s0 != s1
    assert changed.sum() == 1 and changed[0, 1, 1]
    same = np.ones(c0.shape, dtype=bool)
    same[0, 64:128, 1, :] = False
    assert np.array_equal(c0[same], c1[same])


def test_granularities_that_must_coincide():
    rng = np.random.default_rng(4)
    x = _bf16_like(rng, (2, 100, 3, 8))
    ch, sh = quant.quantize_blockwise(x, "e4m3", "per_head")
    ct, st = quant.quantize_blockwise(x, "e4m3", "per_token_block", 128)  # one block covers all rows
    assert np.array_equal(ch, ct) and np.array_equal(sh, st[:, :, 0])
    x1 = x[:1, :, :1, :]
    c1, s1 = quant.quantize_blockwise(x1, "int8", "per_head")
    c2, s2 = quant.quantize_blockwise(x1, "int8", "per_tensor")
    assert np.array_equal(c1, c2) and s1[0, 0] == s2[0]
    xd = x[:, :, :, :1]
    c3, s3 = quant.quantize_blockwise(xd, "int8", "per_channel")
    c4, s4 = quant.quantize_blockwise(xd, "int8", "per_head")
    assert np.array_equal(c3, c4) and np.array_equal(s3[:, :, 0], s4)


def test_e4m3_division_matches_torch_rounding():
    # The element code is RN(x / scale) computed in float32; torch's own
    # float8 conversion of the same float32 quotient must agree.
    import torch

    rng = np.random.default_rng(5)
    x = _bf16_like(rng, (1, 512, 1, 64), 3.0)
    codes, scales = quant.quantize_blockwise(x, "e4m3", "per_tensor")
    q = (x / scales[0]).astype(np.float32)
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def _rn32(fr):
    """The float32 nearest to a positive rational, ties to even, exactly."""
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(0)), f, np.nextafter(f, np.float32(np.inf))]
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - fr), int(np.float32(c).view(np.uint32)) & 1))


@pytest.mark.parametrize("out", ["int8", "e4m3"])
def test_scale_is_the_correctly_rounded_quotient(out):
    """scale = RN(amax / R): for every positive finite BF16 amax, the float32
    nearest to the exact rational amax / R (a multiplication by a rounded
    reciprocal differs on some of them)."""
    amax = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    R = int(quant.RANGE[out])
    got = quant.scale_from_amax(amax, out)
    want = np.array([_rn32(Fraction(float(a)) / R) for a in amax], dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("first_dominates", [True, False])
def test_token_block_extent(first_dominates):
    """Each token block covers exactly its rows: every block holds a spike in its
    first and in its last row, and the dominant spike grows (first rows) or
    shrinks (last rows) from block to block, so a block that reaches one row
    into a neighbour, or stops one row short, takes a different amax. S = 200
    with 64-row blocks leaves a ragged last block of 8 rows."""
    rng = np.random.default_rng(6)
    S, rpb, nblk = 200, 64, 4
    x = (rng.uniform(-1.0, 1.0, size=(1, S, 2, 8))).astype(np.float32)
    want = np.zeros((1, 2, nblk), dtype=np.float32)
    for i in range(nblk):
        first, last = i * rpb, min(S, (i + 1) * rpb) - 1
        big = np.float32(10.0 * 4.0 ** i) if first_dominates else np.float32(10.0 * 4.0 ** (nblk - i))
        x[0, first, :, 3] = big if first_dominates else big / 2
        x[0, last, :, 5] = -(big / 2) if first_dominates else -big
        want[0, :, i] = big
    codes, scales = quant.quantize_blockwise(x, "int8", "per_token_block", rpb)
    assert np.array_equal(scales, quant.scale_from_amax(want, "int8"))
