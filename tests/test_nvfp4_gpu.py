"""Per-token NVFP4 quantizer (fmha_quantize_nvfp4) against the oracle: codes,
E4M3 block scales and fp32 token scales bit for bit ("FlashInfer per-token
NVFP4 quantization kernel")."""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import nvfp4 as on
from precision_attention_fmha_b200 import fmha

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def make_rows(seed, rows, K, scale=1.0, outliers=0.01):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, K)) * scale).astype(np.float32)
    x[rng.random((rows, K)) < outliers] *= 40
    return torch.from_numpy(x).to(torch.bfloat16)


def check(x_bf16, fast, rows_sample=None, src_view=None):
    xg = (src_view if src_view is not None else x_bf16).to(DEV) if src_view is None else src_view
    codes, sb, st = fmha.quantize_nvfp4(xg, fast_math=fast)
    fmha.get_device_error()
    x32 = x_bf16.to(torch.float32).numpy()
    idx = np.arange(x32.shape[0]) if rows_sample is None else rows_sample
    rc, rsb, rst = on.quantize_per_token(x32[idx], fast_math=fast)
    assert np.array_equal(st.cpu().numpy()[idx].view(np.uint32), rst.view(np.uint32))
    assert np.array_equal(sb.view(torch.uint8).cpu().numpy()[idx], rsb)
    assert np.array_equal(codes.cpu().numpy()[idx], rc)


@pytest.mark.parametrize("fast", [False, True])
@pytest.mark.parametrize("rows,K", [(1, 16), (3, 48), (257, 256), (64, 4096), (5, 16384), (2, 2064)])
def test_bit_exact(rows, K, fast):
    check(make_rows(rows * 7 + K, rows, K), fast)


@pytest.mark.parametrize("fast", [False, True])
def test_small_and_wide_range_rows(fast):
    x = make_rows(11, 6, 512, scale=1e-3, outliers=0.05)
    x[1] = 0                      # zero row: token scale 1, everything zero
    x[2, :256] = 0                # zero blocks
    x[3] *= 1e4                   # large values
    x[4, ::7] = -x[4, ::7]
    check(x, fast)


def test_strided_source_rows():
    base = make_rows(13, 33, 1024 + 64)
    view = base.to(DEV)[:, :1024]          # row stride 1088 elements
    check(base[:, :1024].contiguous(), False, src_view=view)


def test_dequantized_error_is_bounded():
    x = make_rows(17, 16, 2048)
    codes, sb, st = fmha.quantize_nvfp4(x.to(DEV))
    xr = on.dequantize(codes.cpu().numpy(), sb.view(torch.uint8).cpu().numpy(), st.cpu().numpy())
    x32 = x.to(torch.float32).numpy()
    e = np.repeat(sb.float().cpu().numpy(), 16, axis=1) * st.cpu().numpy()[:, None]
    assert np.all(np.abs(x32 - xr) <= e * (1 + 1e-6))


@pytest.mark.big
def test_full_size_sampled_rows():
    """16384 tokens x 4096: the GPU result for sampled rows equals the oracle's."""
    x = make_rows(19, 16384, 4096)
    rows = np.unique(np.concatenate([[0, 1, 8191, 16383], np.random.default_rng(3).integers(0, 16384, 28)]))
    check(x, False, rows_sample=rows)


@pytest.mark.parametrize("fast", [False, True])
def test_elements_at_rounding_midpoints(fast):
    """Values whose scaled value x / e falls on or next to an E2M1 rounding
    midpoint (0.25, 0.75, ..., 5): the exact path must still round RN(x / e)."""
    rng = np.random.default_rng(23)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for A in (6.0, 3.0, 0.1875, 448.0, 1.0 / 3.0, 1234.5):
        a = np.float32(ml_dtypes.bfloat16(A))
        s_t = np.float32(a / np.float32(2688.0))
        q = np.float32(np.float32(a / s_t) / np.float32(6.0))
        from oracle import e4m3
        sb = e4m3.decode(e4m3.encode(np.array([q])))[0]
        e = np.float32(np.float32(sb) * s_t)
        for _ in range(4):
            row = np.zeros(256, dtype=np.float32)
            row[0] = a
            m = rng.choice(mids, 255) * rng.choice([-1.0, 1.0], 255)
            jitter = 1 + rng.choice([-2.0 ** -8, 0.0, 2.0 ** -8], 255)  # one BF16 step either side, or none
            row[1:] = (m * e * jitter).astype(np.float32)
            rows.append(row)
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    check(x, fast)
