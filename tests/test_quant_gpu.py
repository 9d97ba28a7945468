"""GPU quantizer vs the oracle: codes and scales bit-exact, every granularity.

Sizes span several CTAs, ragged token blocks and the grid-wide reductions;
the workload-sized cases run under -m "gpu and big"."""

import numpy as np
import pytest
import torch

from oracle import quant as oq
from precision_attention_fmha_b200 import fmha, workloads
from tests.helpers import codes_np, f32

pytestmark = pytest.mark.gpu

DT = {"int8": torch.int8, "e4m3": torch.float8_e4m3fn}


def _check(x_bf16, out, kind, rpb):
    dev = torch.device("cuda")
    codes, scales = fmha.fmha_quantize_blockwise(x_bf16.to(dev), DT[out], kind, rpb)
    torch.cuda.synchronize()
    ref_c, ref_s = oq.quantize_blockwise(f32(x_bf16), out, kind, rpb)
    got_c = codes_np(codes)
    got_s = scales.cpu().numpy().reshape(ref_s.shape)
    assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32)), "scales differ"
    mism = np.count_nonzero(got_c != ref_c)
    assert mism == 0, f"{mism} codes differ of {got_c.size}"


@pytest.mark.parametrize("out", ["int8", "e4m3"])
@pytest.mark.parametrize("kind,rpb", [("per_token_block", 128), ("per_token_block", 64), ("per_token_block", 200),
                                      ("per_head", None), ("per_tensor", None), ("per_channel", None)])
@pytest.mark.parametrize("S", [1, 77, 384, 1000])
def test_quantizer_bit_exact(out, kind, rpb, S):
    B, H, D = 2, 3, 128
    q, _, _ = workloads.biased_qk_v(50 + S, B, S, H, D)
    _check(q, out, kind, rpb)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_quantizer_head_dims(D):
    x, _, _ = workloads.outlier_qkv(60 + D, 1, 300, 2, D)
    for kind, rpb in (("per_token_block", 64), ("per_channel", None), ("per_head", None)):
        _check(x, "e4m3", kind, rpb)


def test_quantizer_strided_view_and_zero_block():
    dev = torch.device("cuda")
    big = torch.zeros(2, 256, 4, 128, dtype=torch.bfloat16)
    big[:, 128:, :, :] = torch.randn(2, 128, 4, 128).to(torch.bfloat16) * 3
    view = big[:, :, 1:3, :]  # non-packed head stride
    codes, scales = fmha.fmha_quantize_blockwise(view.to(dev), torch.int8, "per_token_block", 128)
    ref_c, ref_s = oq.quantize_blockwise(f32(view), "int8", "per_token_block", 128)
    assert np.array_equal(codes_np(codes), ref_c)
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    assert np.all(scales.cpu().numpy()[:, :, 0] == 1.0)


@pytest.mark.big
@pytest.mark.parametrize("name", ["sage_q", "sage_k", "sage_v", "fp8_q", "pv8_v"])
def test_quantizer_workload_sizes(name):
    if name.startswith("sage"):
        q, k, v = workloads.biased_qk_v(workloads.SEED_BASE + 4 + 16384, 1, 16384, 24, 128)
        x, out, kind, rpb = {"sage_q": (q, "int8", "per_token_block", 128),
                             "sage_k": (k, "int8", "per_token_block", 64),
                             "sage_v": (v, "e4m3", "per_channel", None)}[name]
    elif name == "fp8_q":
        x, _, _ = workloads.outlier_qkv(workloads.SEED_BASE + 3 + 8192, 2, 8192, 32, 128)
        out, kind, rpb = "e4m3", "per_head", None
    else:
        _, _, x = workloads.normal_qkv(workloads.SEED_BASE + 2 + 16384, 1, 16384, 16384, 40, 40, 128)
        out, kind, rpb = "e4m3", "per_tensor", None
    _check(x, out, kind, rpb)


@pytest.mark.parametrize("out", ["int8", "e4m3"])
@pytest.mark.parametrize("kind,rpb", [("per_token_block", 64), ("per_head", None), ("per_tensor", None),
                                      ("per_channel", None)])
def test_quantizer_empty_sequence(out, kind, rpb):
    """S == 0: no code is written; the grid-wide kinds write scale 1.0 (amax 0) into every group."""
    B, H, D = 2, 3, 128
    x = torch.zeros((B, 0, H, D), dtype=torch.bfloat16)
    ref_c, ref_s = oq.quantize_blockwise(f32(x), out, kind, rpb)
    dev = torch.device("cuda")
    scales = torch.full(fmha.scale_shape(kind, B, 0, H, D, rpb), float("nan"), device=dev)
    codes, scales = fmha.fmha_quantize_blockwise(x.to(dev), DT[out], kind, rpb, scales=scales)
    torch.cuda.synchronize()
    assert codes.numel() == 0
    got_s = scales.cpu().numpy().reshape(ref_s.shape)
    assert np.array_equal(got_s, ref_s)
    if kind != "per_token_block":
        assert np.all(got_s == 1.0)
