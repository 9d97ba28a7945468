"""Pins for the NVFP4 oracle (oracle/nvfp4.py): the E2M1 codec against the
format's value table (tests/golden/e2m1_spec_values.txt) and an independent
encoder (ml_dtypes), and the per-token recipe against properties that the
two-level scale fixes ("FlashInfer per-token NVFP4 quantization kernel")."""

import os

import ml_dtypes
import numpy as np
import pytest

from oracle import e4m3, nvfp4

HERE = os.path.dirname(__file__)


def golden():
    rows = []
    with open(os.path.join(HERE, "golden", "e2m1_spec_values.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                c, v = line.split()
                rows.append((int(c), float(v)))
    return rows


def test_decode_matches_spec_table():
    for c, v in golden():
        got = nvfp4.e2m1_decode(np.array([c]))[0]
        assert got == v and np.signbit(got) == np.signbit(v), (c, got, v)


def test_encode_round_trips_every_code():
    for c, v in golden():
        assert nvfp4.e2m1_encode(np.array([v]))[0] == c


@pytest.mark.parametrize("x,code", [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
                                    (0.2499, 0), (0.2501, 1), (2.51, 5), (5.01, 7), (7.0, 7), (1e9, 7),
                                    (-0.75, 10), (-5.0, 14), (-100.0, 15)])
def test_ties_to_even_and_saturation(x, code):
    assert nvfp4.e2m1_encode(np.array([x]))[0] == code


def test_encode_agrees_with_an_independent_encoder():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-8, 8, 200000), rng.standard_normal(100000) * 3,
                        np.arange(-14, 14.001, 0.125)]).astype(np.float32)
    ours = nvfp4.e2m1_decode(nvfp4.e2m1_encode(x))
    ref = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ours, ref)


def rows_bf16(seed, rows, K, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, K)) * scale).astype(np.float32)
    hit = rng.random((rows, K)) < 0.01  # a few outliers
    x[hit] *= 30
    return x.astype(ml_dtypes.bfloat16).astype(np.float32)


@pytest.mark.parametrize("fast", [False, True])
def test_token_and_block_scales(fast):
    x = rows_bf16(1, 5, 256)
    packed, sb, st = nvfp4.quantize_per_token(x, fast_math=fast)
    amax = np.abs(x).max(axis=1).astype(np.float32)
    assert np.array_equal(st, (amax / np.float32(2688.0)).astype(np.float32))
    for r in range(x.shape[0]):
        j = int(np.argmax(np.abs(x[r]))) // 16  # the block holding the row's amax
        assert abs(e4m3.decode(np.array([sb[r, j]]))[0] - 448.0) <= 16.0  # one E4M3 step at 448
        c = np.concatenate([packed[r] & 0xF, packed[r] >> 4])  # codes of the row (any order)
        assert np.any((c & 7) == 7)  # the amax element lands on the largest E2M1 magnitude


@pytest.mark.parametrize("fast", [False, True])
def test_each_code_brackets_its_scaled_value(fast):
    """Every code is one of the two E2M1 values around x / e (or +-6 above 6)."""
    x = rows_bf16(2, 4, 512, scale=0.01)
    packed, sb, st = nvfp4.quantize_per_token(x, fast_math=fast)
    codes = np.zeros(x.shape, dtype=np.uint8)
    codes[:, 0::2], codes[:, 1::2] = packed & 0xF, packed >> 4
    e = np.repeat(e4m3.decode(sb), 16, axis=1) * st.astype(np.float64)[:, None]
    grid = np.sort(np.unique(np.abs(nvfp4.e2m1_decode(np.arange(8)))))
    y = np.abs(x / np.where(e == 0, 1, e))
    val = np.abs(nvfp4.e2m1_decode(codes))
    lo = grid[np.clip(np.searchsorted(grid, y, side="right") - 1, 0, 7)]
    hi = grid[np.clip(np.searchsorted(grid, y, side="left"), 0, 7)]
    ok = (val == lo) | (val == hi) | (e == 0)
    assert ok.all()
    assert np.array_equal(np.signbit(nvfp4.e2m1_decode(codes)) & (val > 0), (x < 0) & (val > 0))


def test_dequantization_error_bound():
    x = rows_bf16(3, 8, 1024)
    packed, sb, st = nvfp4.quantize_per_token(x)
    xr = nvfp4.dequantize(packed, sb, st)
    e = np.repeat(e4m3.decode(sb), 16, axis=1) * st.astype(np.float64)[:, None]
    # largest E2M1 gap is 2 (between 4 and 6): |x - x^| <= e (plus fp32 rounding of x / e)
    assert np.all(np.abs(x - xr) <= e * (1 + 1e-6) + 1e-30)


def test_zero_rows_and_blocks():
    x = np.zeros((2, 64), dtype=np.float32)
    x[1, 16:32] = 3.0
    packed, sb, st = nvfp4.quantize_per_token(x)
    assert st[0] == 1.0 and np.all(sb[0] == 0) and np.all(packed[0] == 0)
    assert np.all(sb[1, [0, 2, 3]] == 0) and np.all(packed[1, :8] == 0) and np.all(packed[1, 16:] == 0)
    assert np.all(nvfp4.dequantize(packed, sb, st)[1, 16:32] == pytest.approx(3.0, rel=2 ** -3))


def test_packing_order():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0], x[0, 1] = 6.0, -3.0  # amax 6: e ~ 1, codes 7 and 13
    packed, sb, st = nvfp4.quantize_per_token(x)
    assert packed[0, 0] == (7 | (13 << 4))


def test_every_block_maps_its_amax_to_six():
    """The block scale is E4M3((amax_blk / s_t) / 6), so each block's largest
    element lands on E2M1's largest magnitude: amax_blk / e = 6 q / decode(E4M3(q))
    lies within 6 (1 +- 2^-4) whenever E4M3(q) is normal, which rounds (or
    saturates) to 6. Blocks whose scale falls into E4M3's subnormal range have
    coarser steps and are left out."""
    x = rows_bf16(4, 16, 1024)
    x *= np.exp2(np.random.default_rng(5).integers(-6, 4, size=(16, 64))).repeat(16, axis=1).astype(np.float32)
    packed, sb, st = nvfp4.quantize_per_token(x)
    codes = np.zeros(x.shape, dtype=np.uint8)
    codes[:, 0::2], codes[:, 1::2] = packed & 0xF, packed >> 4
    mags = np.abs(nvfp4.e2m1_decode(codes)).reshape(16, 64, 16).max(axis=2)
    normal = e4m3.decode(sb) >= 2.0 ** -6
    assert normal.sum() > 500
    assert np.all(mags[normal] == 6.0)
