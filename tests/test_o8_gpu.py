"""E4M3 output (o = E4M3(O / sf_o)) against the oracle, for every dtype tuple.

The kernel's fp32 O differs from the oracle's fp64 O by the attention error,
so the codes cannot be compared bit for bit. The bound follows from the
arithmetic instead. E4M3 keeps 3 mantissa bits, so round-to-nearest moves a
normal value by at most 2^-4 of its magnitude, and a subnormal (step 2^-9)
by at most 2^-10. Hence, per element,
    |decode(code) * sf_o - O_ref| <= 2^-4 |O_ref| + 2^-10 sf_o + atol,
where atol is the tuple's own attention tolerance. The per-head cosine takes
the rounding's share, at most about (2^-4)^2 / 6 ~ 7e-4 of 1 - cos. Measured
1 - cos stays below 7.0e-4 for every tuple (5e-4 on these shapes), so every
tuple is held to the attention's own per-head bound, cos >= 0.999.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import e4m3 as oe
from precision_attention_fmha_b200 import fmha, workloads
from precision_attention_fmha_b200.fmha import Scale
from tests.helpers import Q8_COS, codes_np, cos_per_head, f64
from tests.test_fmha_gpu import prepare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
E4M3 = torch.float8_e4m3fn
MAX_E4M3_CODE = {0x7E, 0xFE}  # +-448


def _inputs(mode, B, Hq, Hkv, Sq, Skv, D, seed):
    if mode == "fp8":
        q, k, v = workloads.outlier_qkv(seed, B, max(Sq, Skv), Hq, D)
        return q[:, :Sq], k[:, :Skv, :Hkv], v[:, :Skv, :Hkv]
    if mode == "sage":
        q, _, _ = workloads.biased_qk_v(seed, B, Sq, Hq, D)
        _, k, v = workloads.biased_qk_v(seed + 1, B, Skv, Hkv, D)
        return q, k, v
    return workloads.normal_qkv(seed, B, Sq, Skv, Hq, Hkv, D)


def _extra(mode, B, Hq, Sq):
    if mode != "sage":
        return {}
    sf_p = Scale(torch.full((B, Hq, math.ceil(Sq / 128)), workloads.SAGE_SF_P, device=DEV), "per_token_block", 128)
    return {"sf_p": sf_p, "p_terms": 1}


def check_o8(codes, sf_o, ref, mode):
    c = codes_np(codes)
    got = oe.decode(c) * sf_o
    assert not np.isnan(got).any(), "NaN code in the output"
    if mode == "bf16":
        atol = 1e-2
    else:  # 8-bit tolerance, scaled per head by the output's magnitude
        atol = 3e-2 * np.maximum(1.0, np.abs(ref).max(axis=(1, 3)))[:, None, :, None]
    bound = 2.0 ** -4 * np.abs(ref) + 2.0 ** -10 * sf_o + atol
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"err {err[worst]:.3e} > bound {np.broadcast_to(bound, err.shape)[worst]:.3e}"
    cos_min = Q8_COS
    cos = cos_per_head(got, ref)
    assert cos.min() >= cos_min, cos.min()


@pytest.mark.parametrize("mode", ["bf16", "pv8", "fp8", "sage"])
@pytest.mark.parametrize("B,Hq,Hkv,Sq,Skv,causal", [
    (1, 4, 2, 300, 300, True),
    (2, 2, 2, 513, 700, False),
    (1, 3, 1, 200, 100, True),   # Sq > Skv causal: leading rows see nothing -> code 0
])
def test_e4m3_output(mode, B, Hq, Hkv, Sq, Skv, causal):
    D = 128
    q, k, v = _inputs(mode, B, Hq, Hkv, Sq, Skv, D, seed=900 + Sq + Skv + B)
    g, rq, rk, rv = prepare(mode, q.contiguous(), k.contiguous(), v.contiguous())
    scale = 1 / math.sqrt(D)
    ref, ref_lse = oa.attention(rq, rk, rv, scale, causal)
    sf_o_val = float(np.float32(max(np.abs(ref).max(), 1e-3) / 256.0))  # the oracle sets the output range
    sf_o = Scale(torch.tensor([sf_o_val], dtype=torch.float32, device=DEV), "per_tensor", 0)
    out = torch.empty((B, Sq, Hq, D), dtype=E4M3, device=DEV)
    lse8 = torch.empty((B, Hq, Sq), dtype=torch.float32, device=DEV)
    fmha.fmha_fwd(g["q"], g["k"], g["v"], out=out, sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"],
                  softmax_scale=scale, causal=causal, lse=lse8, sf_o=sf_o, **_extra(mode, B, Hq, Sq))
    fmha.get_device_error()
    check_o8(out, sf_o_val, ref, mode)
    dead = ~np.isfinite(ref_lse)  # [B, Hq, Sq] rows with no visible key
    if dead.any():
        c = codes_np(out)
        assert np.all(c.transpose(0, 2, 1, 3)[dead] == 0)
    # The epilogue is the only difference from the BF16-output kernel, so the
    # log-sum-exp agrees with that kernel's (to fp32 rounding).
    lse16 = torch.empty_like(lse8)
    fmha.fmha_fwd(g["q"], g["k"], g["v"], sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"], softmax_scale=scale,
                  causal=causal, lse=lse16, **_extra(mode, B, Hq, Sq))
    fmha.get_device_error()
    assert torch.equal(torch.isfinite(lse8), torch.isfinite(lse16))
    fin = torch.isfinite(lse16)
    assert torch.allclose(lse8[fin], lse16[fin], rtol=1e-6, atol=1e-6)


def test_e4m3_output_default_scale_and_saturation():
    # sf_o NONE means 1.0; outputs beyond 448 saturate to +-448 (no NaN codes).
    B, Hq, Hkv, S, D = 1, 2, 2, 256, 128
    q, k, v = workloads.normal_qkv(950, B, S, S, Hq, Hkv, D)
    v = (v.float() * 2000).to(torch.bfloat16)  # |O| reaches well past 448
    ref, _ = oa.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(D))
    out = torch.empty((B, S, Hq, D), dtype=E4M3, device=DEV)
    fmha.fmha_fwd(q.to(DEV), k.to(DEV), v.to(DEV), out=out)
    fmha.get_device_error()
    c = codes_np(out)
    assert not np.isnan(oe.decode(c)).any()
    big = np.abs(ref) > 448 * (1 + 2.0 ** -4) + 10.0  # clearly beyond the range, whatever the rounding
    assert big.any()
    assert set(np.unique(c[big]).tolist()) <= MAX_E4M3_CODE
    # In range, sf_o = 1: the rounding bound plus the BF16 tolerance scaled
    # with V (x 2000).
    small = np.abs(ref) < 400
    got = oe.decode(c[small])
    assert np.all(np.abs(got - ref[small]) <= 2.0 ** -4 * np.abs(ref[small]) + 2.0 ** -10 + 1e-2 * 2000)


def test_e4m3_output_block_sparse_and_paged():
    B, Hq, Hkv, S, D = 2, 4, 2, 1000, 128
    w = workloads.sparse_paged(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D, page_size=64)
    mask = w["mask"]
    kk = oa.gather_paged(f64(w["k_pool"]), w["page_table"].numpy(), S)
    vv = oa.gather_paged(f64(w["v_pool"]), w["page_table"].numpy(), S)
    ref, _ = oa.attention(f64(w["q"]), kk, vv, w["scale"], False, mask.numpy())
    sf_o_val = float(np.float32(np.abs(ref).max() / 256.0))
    sf_o = Scale(torch.tensor([sf_o_val], dtype=torch.float32, device=DEV), "per_tensor", 0)
    o_paged = torch.empty((B, S, Hq, D), dtype=E4M3, device=DEV)
    fmha.fmha_fwd_paged(w["q"].to(DEV), w["k_pool"].to(DEV), w["v_pool"].to(DEV), w["page_table"].to(DEV), S,
                        mask=mask.to(DEV), out=o_paged, sf_o=sf_o)
    o_sparse = torch.empty_like(o_paged)
    fmha.fmha_fwd_block_sparse(w["q"].to(DEV), w["k"].to(DEV), w["v"].to(DEV), mask.to(DEV), out=o_sparse,
                               sf_o=sf_o)
    fmha.get_device_error()
    check_o8(o_paged, sf_o_val, ref, "bf16")
    assert torch.equal(o_paged.view(torch.uint8), o_sparse.view(torch.uint8))
