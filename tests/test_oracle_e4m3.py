"""Pins for the oracle's E4M3 codec (CPU only).

Pinned against: the OCP OFP8 spec table (golden file), exhaustive round trips
over all 256 codes, hand-built rounding ties, saturation, and two independent
library encoders (ml_dtypes and torch) on a dense sweep.
"""

import os

import numpy as np
import pytest

from oracle import e4m3

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spec_values.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, val = line.split()
            rows.append((int(code, 16), float(val)))
    return rows


def test_spec_table_decode_and_encode():
    for code, val in _golden():
        got = e4m3.decode(np.array([code], dtype=np.uint8))[0]
        if np.isnan(val):
            assert np.isnan(got)
            continue
        assert got == val and np.signbit(got) == np.signbit(val), (hex(code), got, val)
        assert e4m3.encode(np.array([val]))[0] == code, hex(code)


def test_roundtrip_every_finite_code():
    codes = e4m3.all_finite_codes()
    assert codes.size == 254
    vals = e4m3.decode(codes)
    assert np.array_equal(e4m3.encode(vals), codes)


def test_values_strictly_increasing_over_positive_codes():
    vals = e4m3.decode(np.arange(0x00, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(vals) > 0)
    assert vals[-1] == 448.0


def test_midpoints_round_to_even():
    pos = e4m3.decode(np.arange(0x00, 0x7F, dtype=np.uint8))  # 0 .. 448
    for c in range(0x7E):
        lo, hi = pos[c], pos[c + 1]
        mid = (lo + hi) / 2  # exact in float64
        even = c if c % 2 == 0 else c + 1
        assert e4m3.encode(np.array([mid]))[0] == even, (c, mid)
        assert e4m3.encode(np.array([-mid]))[0] == (even | 0x80)
        # a hair either side of the midpoint goes to the nearer code
        eps = (hi - lo) * 1e-6
        assert e4m3.encode(np.array([mid - eps]))[0] == c
        assert e4m3.encode(np.array([mid + eps]))[0] == c + 1


@pytest.mark.parametrize("x", [448.0, 448.5, 464.0, 479.99, 480.0, 512.0, 1e6, 3.4e38])
def test_saturates_to_max_finite(x):
    assert e4m3.encode(np.array([x]))[0] == 0x7E
    assert e4m3.encode(np.array([-x]))[0] == 0xFE


def test_tiny_values_flush_and_round():
    step = 2.0 ** -9
    assert e4m3.encode(np.array([step / 2]))[0] == 0x00  # tie to even -> 0
    assert e4m3.encode(np.array([step * 0.5000001]))[0] == 0x01
    assert e4m3.encode(np.array([step * 1.5]))[0] == 0x02  # tie 1.5 -> 2 (even)
    assert e4m3.encode(np.array([1e-30]))[0] == 0x00


def test_dense_sweep_matches_ml_dtypes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.uniform(-448, 448, 200000),
        rng.normal(0, 1, 200000) * np.exp2(rng.integers(-12, 8, 200000)),
    ]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ours = e4m3.encode(x)
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, ref)


def test_dense_sweep_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(8)
    x = (rng.normal(0, 1, 200000) * np.exp2(rng.integers(-12, 8, 200000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3.encode(x), ref)
