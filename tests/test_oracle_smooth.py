"""Pins for the oracle's K smoothing (token mean per channel, shifted quantizer).

CPU only. A wrong reduction axis, a wrong sign of the shift, a shift applied
after the amax, or a mean rounded twice must fail one of these:

* the mean against a correctly rounded brute-force sum (``math.fsum``);
* a closed form, where constant-plus-alternating data has a known mean;
* quantizing x + c with shift c, where the sum and the difference are exact,
  gives the codes of x;
* a zero shift leaves every granularity unchanged;
* exact attention ignores a per-(b, h, d) shift of K, and its log-sum-exp
  moves by softmax_scale * q . mean (the reason the step exists);
* on keys with a per-channel bias (the SageAttention workload's N(0, 2)
  bias), INT8 attention after smoothing is closer to the exact result.
"""

import math

import numpy as np
import pytest

from oracle import attention as oatt
from oracle import quant


def _bf16_like(rng, shape, scale=1.0, loc=0.0):
    import torch

    x = torch.from_numpy((rng.standard_normal(shape) * scale + loc).astype(np.float32))
    return x.to(torch.bfloat16).to(torch.float32).numpy()


def test_channel_mean_matches_fsum_brute_force():
    rng = np.random.default_rng(11)
    x = _bf16_like(rng, (2, 37, 3, 8), scale=3.0, loc=0.5)
    got = quant.channel_mean(x)
    B, S, H, D = x.shape
    for b in range(B):
        for h in range(H):
            for d in range(D):
                want = np.float32(math.fsum(float(x[b, s, h, d]) for s in range(S)) / S)
                assert got[b, h, d] == want, (b, h, d)
    assert got.dtype == np.float32 and got.shape == (B, H, D)


def test_channel_mean_closed_form():
    # x[s] = c + (-1)^s * e with S even: the e terms cancel, the mean is c.
    B, S, H, D = 1, 64, 2, 4
    c = np.array([[0.75, -3.5, 12.0, 0.0], [1.0 / 1024, -0.25, 5.5, -100.0]], dtype=np.float32)
    e = np.array([[0.5, 2.0, 0.125, 7.0], [0.0, 1.0, 64.0, 0.5]], dtype=np.float32)
    sign = np.where(np.arange(S) % 2 == 0, 1.0, -1.0).astype(np.float32)
    x = c[None, None] + sign[None, :, None, None] * e[None, None]
    np.testing.assert_array_equal(quant.channel_mean(x)[0], c)


def test_channel_mean_axis_is_tokens():
    # Distinct constant per (b, h, d), varying nothing over s: the mean is it.
    x = np.zeros((2, 5, 3, 4), dtype=np.float32)
    for b in range(2):
        for h in range(3):
            for d in range(4):
                x[b, :, h, d] = 100 * b + 10 * h + d
    m = quant.channel_mean(x)
    for b in range(2):
        for h in range(3):
            for d in range(4):
                assert m[b, h, d] == 100 * b + 10 * h + d


def test_channel_mean_keeps_small_terms_next_to_large_ones():
    """The sum is taken in float64: +-2^20 around 2^-10 terms (30 binades apart,
    exact in float64, lost in a float32 running sum) leave the small terms' mean,
    the correctly rounded fsum over S."""
    S = 40
    col = np.full(S, 2.0 ** -10, dtype=np.float32)
    col[0], col[-1] = 2.0 ** 20, -(2.0 ** 20)  # first and last: a running sum holds 2^20 throughout
    col[7] = np.float32(3.0 * 2.0 ** -9)
    x = np.zeros((1, S, 1, 2), dtype=np.float32)
    x[0, :, 0, 0] = col
    x[0, :, 0, 1] = -col
    want = np.float32(math.fsum(float(c) for c in col) / S)
    m = quant.channel_mean(x)[0, 0]
    assert m[0] == want and m[1] == -want and want > 0


def test_channel_mean_empty():
    assert np.all(quant.channel_mean(np.zeros((1, 0, 2, 8), np.float32)) == 0)


@pytest.mark.parametrize("out_dtype", ["int8", "e4m3"])
@pytest.mark.parametrize("kind,rpb", [("per_tensor", None), ("per_head", None), ("per_token_block", 64),
                                      ("per_channel", None)])
def test_zero_shift_is_identity(out_dtype, kind, rpb):
    rng = np.random.default_rng(12)
    x = _bf16_like(rng, (2, 100, 2, 16))
    c0, s0 = quant.quantize_blockwise(x, out_dtype, kind, rpb)
    c1, s1 = quant.quantize_blockwise(x, out_dtype, kind, rpb, shift=np.zeros((2, 2, 16), np.float32))
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(s0, s1)


@pytest.mark.parametrize("out_dtype", ["int8", "e4m3"])
@pytest.mark.parametrize("kind,rpb", [("per_head", None), ("per_token_block", 32), ("per_channel", None)])
def test_shift_is_subtracted(out_dtype, kind, rpb):
    # x holds BF16 values with |x| >= 2^-10 (or 0), c is a power of two per
    # (b, h, d), |c| <= 8: x + c and (x + c) - c are exact in float32, so the
    # shifted quantization of x + c must give x's own codes and scales. A shift
    # added instead of subtracted gives x + 2c and fails.
    rng = np.random.default_rng(13)
    B, S, H, D = 2, 96, 2, 16
    x = _bf16_like(rng, (B, S, H, D))
    x[np.abs(x) < 2.0 ** -10] = 0.0
    c = (2.0 ** rng.integers(-2, 4, size=(B, H, D)) * rng.choice([-1.0, 1.0], size=(B, H, D))).astype(np.float32)
    xc = (x + c[:, None]).astype(np.float32)
    assert np.array_equal((xc - c[:, None]).astype(np.float32), x)
    c0, s0 = quant.quantize_blockwise(x, out_dtype, kind, rpb)
    c1, s1 = quant.quantize_blockwise(xc, out_dtype, kind, rpb, shift=c)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(s0, s1)
    c2, _ = quant.quantize_blockwise(xc, out_dtype, kind, rpb)
    assert not np.array_equal(c0, c2)


def test_shift_shape_checked():
    with pytest.raises(ValueError):
        quant.quantize_blockwise(np.zeros((1, 4, 2, 8), np.float32), "int8", "per_head", shift=np.zeros((2, 8)))


@pytest.mark.parametrize("causal", [False, True])
def test_exact_attention_ignores_k_mean(causal):
    rng = np.random.default_rng(14)
    B, Sq, Skv, Hq, Hkv, D = 1, 40, 40, 4, 2, 16
    q = rng.standard_normal((B, Sq, Hq, D))
    k = rng.standard_normal((B, Skv, Hkv, D)) + 3.0 * rng.standard_normal((B, 1, Hkv, D))
    v = rng.standard_normal((B, Skv, Hkv, D))
    scale = 1.0 / math.sqrt(D)
    mu = quant.channel_mean(k.astype(np.float32)).astype(np.float64)  # [B, Hkv, D]
    o0, lse0 = oatt.attention(q, k, v, scale, causal=causal)
    o1, lse1 = oatt.attention(q, k - mu[:, None], v, scale, causal=causal)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    group = Hq // Hkv
    for h in range(Hq):
        shift = scale * q[0, :, h, :] @ mu[0, h // group]  # [Sq]
        np.testing.assert_allclose(lse1[0, h], lse0[0, h] - shift, rtol=0, atol=1e-11)


def test_smoothing_reduces_int8_attention_error_on_biased_keys():
    # The SageAttention workload's keys: N(0, 1) plus a per-(h, d) bias N(0, 2),
    # INT8 in 64-token blocks. Removing the bias shrinks every block's amax, so
    # the scales (the quantization steps) and the error of attention computed
    # on the dequantized keys both fall. Q stays exact to isolate K's error.
    rng = np.random.default_rng(15)
    B, S, H, D = 1, 256, 4, 64
    bias_q = rng.standard_normal((1, 1, H, D)) * math.sqrt(2.0)
    bias_k = rng.standard_normal((1, 1, H, D)) * math.sqrt(2.0)
    q = _bf16_like(rng, (B, S, H, D)) + bias_q.astype(np.float32)
    k = _bf16_like(rng, (B, S, H, D)) + bias_k.astype(np.float32)
    v = _bf16_like(rng, (B, S, H, D))
    scale = 1.0 / math.sqrt(D)
    o_exact, _ = oatt.attention(q, k, v, scale)
    ck, sk = quant.quantize_blockwise(k, "int8", "per_token_block", 64)
    k_hat = quant.dequantize(ck, sk, "int8", "per_token_block", 64)
    mu = quant.channel_mean(k)
    cks, sks = quant.quantize_blockwise(k, "int8", "per_token_block", 64, shift=mu)
    ks_hat = quant.dequantize(cks, sks, "int8", "per_token_block", 64)
    # Smoothed codes dequantize to k - mean within half a step of each block.
    step = np.repeat(sks, 64, axis=2)[:, :, :S].transpose(0, 2, 1)[..., None]
    assert np.all(np.abs(ks_hat - (k - mu[:, None])) <= step / 2 + 1e-12)
    assert sks.mean() < 0.75 * sk.mean(), (sks.mean(), sk.mean())
    e_plain = oatt.attention(q, k_hat, v, scale)[0] - o_exact
    e_smooth = oatt.attention(q, ks_hat, v, scale)[0] - o_exact
    rms = lambda e: float(np.sqrt(np.mean(e * e)))  # noqa: E731
    assert rms(e_smooth) < 0.8 * rms(e_plain), (rms(e_smooth), rms(e_plain))
