"""K smoothing on the GPU (token mean per channel, shifted quantizer) against the oracle.

* The channel mean is bit-exact where the fp64 sum is exact. Inputs whose
  magnitudes span at most 2^45 / S make it so: BF16 data with every
  |x| < 2^-20 set to 0. On unclamped data it is within one float32 ulp.
* The shifted quantizer is bit-exact, given the same shift. The shift fed to
  both sides is the ORACLE's mean, so no expected value comes from the GPU.
* The Sage attention path on smoothed K matches the oracle on the dequantized
  smoothed operands with the 8-bit tolerance. On biased keys it is closer to
  exact BF16 attention than the same path without smoothing.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import quant as oq
from precision_attention_fmha_b200 import fmha, workloads
from precision_attention_fmha_b200.fmha import Scale
from tests.helpers import assert_close_q8, codes_np, f32, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
DT = {"int8": torch.int8, "e4m3": torch.float8_e4m3fn}


def _clamp_small(x, limit=2.0 ** -20):
    x = x.clone()
    x[x.abs() < limit] = 0
    return x


def _ulp_diff(a, b):
    ia = a.view(np.int32).astype(np.int64)
    ib = b.view(np.int32).astype(np.int64)
    ia = np.where(ia < 0, -(ia & 0x7FFFFFFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFFFFFF), ib)
    return np.abs(ia - ib)


@pytest.mark.parametrize("B,S,H,D", [(2, 1000, 3, 128), (1, 37, 2, 64), (1, 128, 1, 128), (2, 300, 2, 256),
                                     (1, 4096, 4, 128), (1, 1, 2, 8)])
def test_channel_mean_bit_exact(B, S, H, D):
    _, k, _ = workloads.biased_qk_v(700 + S + D, B, S, H, D)
    k = _clamp_small(k)
    got = fmha.channel_mean(k.to(DEV)).cpu().numpy()
    want = oq.channel_mean(f32(k))
    assert got.shape == want.shape
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), int((got != want).sum())


def test_channel_mean_unclamped_within_one_ulp():
    _, k, _ = workloads.biased_qk_v(711, 1, 16384, 4, 128)
    got = fmha.channel_mean(k.to(DEV)).cpu().numpy()
    want = oq.channel_mean(f32(k))
    assert _ulp_diff(got, want).max() <= 1


def test_channel_mean_strided_view_and_empty():
    _, base, _ = workloads.biased_qk_v(712, 2, 200, 5, 128)
    view = _clamp_small(base)[:, :, 1:4, :]  # head stride 128, token stride 640
    got = fmha.channel_mean(view.to(DEV)).cpu().numpy()
    assert np.array_equal(got, oq.channel_mean(f32(view)))
    empty = torch.zeros(1, 0, 2, 64, dtype=torch.bfloat16, device=DEV)
    assert torch.all(fmha.channel_mean(empty) == 0)


@pytest.mark.parametrize("out", ["int8", "e4m3"])
@pytest.mark.parametrize("kind,rpb", [("per_token_block", 64), ("per_token_block", 128), ("per_token_block", 200),
                                      ("per_head", None), ("per_tensor", None), ("per_channel", None)])
@pytest.mark.parametrize("S", [77, 1000])
def test_shifted_quantizer_bit_exact(out, kind, rpb, S):
    B, H, D = 2, 3, 128
    _, k, _ = workloads.biased_qk_v(720 + S, B, S, H, D)
    shift = oq.channel_mean(f32(k))  # the oracle's mean, fed to both sides
    codes, scales = fmha.fmha_quantize_blockwise(k.to(DEV), DT[out], kind, rpb,
                                                 shift=torch.from_numpy(shift).to(DEV))
    rc, rs = oq.quantize_blockwise(f32(k), out, kind, rpb, shift=shift)
    assert np.array_equal(scales.cpu().numpy().reshape(rs.shape).view(np.uint32), rs.view(np.uint32))
    assert np.count_nonzero(codes_np(codes) != rc) == 0


def test_quantize_smoothed_matches_oracle_pipeline():
    # The one-call path: GPU mean -> GPU shifted quantizer. The means agree bit
    # for bit on these (clamped) inputs, so the codes must too.
    _, k, _ = workloads.biased_qk_v(730, 1, 2048, 4, 128)
    k = _clamp_small(k)
    codes, scales, mean = fmha.quantize_smoothed(k.to(DEV), torch.int8, "per_token_block", 64)
    rm = oq.channel_mean(f32(k))
    rc, rs = oq.quantize_blockwise(f32(k), "int8", "per_token_block", 64, shift=rm)
    assert np.array_equal(mean.cpu().numpy(), rm)
    assert np.array_equal(codes_np(codes), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)


def _sage_attention(q, k, v, smooth, causal):
    """GPU Sage path (INT8 Q/K, E4M3 per-channel V) and its oracle operands. P is split
    into two E4M3 terms here: the comparison with and without smoothing measures the INT8
    K error, so the P rounding noise is kept well below it."""
    qc, qs = fmha.fmha_quantize_blockwise(q.to(DEV), torch.int8, "per_token_block", 128)
    if smooth:
        shift = oq.channel_mean(f32(k))
        kc, ks = fmha.fmha_quantize_blockwise(k.to(DEV), torch.int8, "per_token_block", 64,
                                              shift=torch.from_numpy(shift).to(DEV))
    else:
        shift = None
        kc, ks = fmha.fmha_quantize_blockwise(k.to(DEV), torch.int8, "per_token_block", 64)
    vc, vs = fmha.fmha_quantize_blockwise(v.to(DEV), torch.float8_e4m3fn, "per_channel")
    B, Sq, Hq, D = q.shape
    sf_p = Scale(torch.full((B, Hq, math.ceil(Sq / 128)), workloads.SAGE_SF_P, device=DEV), "per_token_block", 128)
    o = fmha.fmha_fwd(qc, kc, vc, sf_q=Scale(qs, "per_token_block", 128), sf_k=Scale(ks, "per_token_block", 64),
                      sf_v=Scale(vs, "per_channel", 0), sf_p=sf_p, softmax_scale=1 / math.sqrt(D),
                      causal=causal, p_terms=2)
    fmha.get_device_error()
    rq = oq.dequantize(*oq.quantize_blockwise(f32(q), "int8", "per_token_block", 128), "int8", "per_token_block", 128)
    rk = oq.dequantize(*oq.quantize_blockwise(f32(k), "int8", "per_token_block", 64, shift=shift), "int8",
                       "per_token_block", 64)
    rv = oq.dequantize(*oq.quantize_blockwise(f32(v), "e4m3", "per_channel"), "e4m3", "per_channel")
    return f64(o), rq, rk, rv


@pytest.mark.parametrize("B,Hq,Hkv,S,causal", [(1, 4, 2, 700, False), (2, 2, 2, 513, True)])
def test_sage_attention_on_smoothed_k(B, Hq, Hkv, S, causal):
    q, _, _ = workloads.biased_qk_v(740 + S, B, S, Hq, 128)
    _, k, v = workloads.biased_qk_v(741 + S, B, S, Hkv, 128)
    o, rq, rk, rv = _sage_attention(q, k, v, True, causal)
    ref, _ = oa.attention(rq, rk, rv, 1 / math.sqrt(128), causal)
    assert_close_q8(o, ref)
    # Exact attention on the original BF16 operands: smoothing must bring the
    # 8-bit path closer to it than the unsmoothed path gets.
    exact, _ = oa.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128), causal)
    o_plain = _sage_attention(q, k, v, False, causal)[0]
    rms = lambda e: float(np.sqrt(np.mean(e * e)))  # noqa: E731
    assert rms(o - exact) < rms(o_plain - exact), (rms(o - exact), rms(o_plain - exact))


@pytest.mark.big
def test_smoothing_sage_workload_size():
    # K of the SageAttention workload: B1 H24 S16384 D128, INT8 in 64-token blocks.
    w = workloads.sage()
    k = w["k"]
    got_mean = fmha.channel_mean(k.to(DEV)).cpu().numpy()
    rm = oq.channel_mean(f32(k))
    assert _ulp_diff(got_mean, rm).max() <= 1
    codes, scales = fmha.fmha_quantize_blockwise(k.to(DEV), torch.int8, "per_token_block", 64,
                                                 shift=torch.from_numpy(rm).to(DEV))
    rc, rs = oq.quantize_blockwise(f32(k), "int8", "per_token_block", 64, shift=rm)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.count_nonzero(codes_np(codes) != rc) == 0
