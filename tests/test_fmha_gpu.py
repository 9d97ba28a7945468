"""GPU attention vs the float64 oracle, element by element.

Each precision mode takes its 8-bit operands from the GPU quantizer, whose
codes and scales are first asserted bit-exact against the oracle quantizer;
the oracle then runs attention on the oracle's dequantized operands. Sizes
span several tiles and CTAs with ragged tails; the edge cases (one token,
Sq != Skv with causal, GQA in both CTA pairings, empty K/V, strided output)
are covered too."""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import quant as oq
from precision_attention_fmha_b200 import fmha, workloads
from precision_attention_fmha_b200.fmha import Scale
from tests.helpers import Q8_ATOL, assert_close_bf16, assert_close_q8, codes_np, f32, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
E4M3 = torch.float8_e4m3fn

# mode -> per-operand (dtype, granularity, rows_per_block) for Q, K, V
MODES = {
    "bf16": None,
    "pv8": {"v": ("e4m3", "per_tensor", None)},
    "fp8": {"q": ("e4m3", "per_head", None), "k": ("e4m3", "per_head", None), "v": ("e4m3", "per_head", None)},
    "sage": {"q": ("int8", "per_token_block", 128), "k": ("int8", "per_token_block", 64),
             "v": ("e4m3", "per_channel", None)},
}
TORCH_DT = {"int8": torch.int8, "e4m3": E4M3}


def quantize_both(x, spec):
    """GPU quantizer output (asserted bit-exact with the oracle) + oracle dequantized values."""
    out, kind, rpb = spec
    codes, scales = fmha.fmha_quantize_blockwise(x.to(DEV), TORCH_DT[out], kind, rpb)
    rc, rs = oq.quantize_blockwise(f32(x), out, kind, rpb)
    assert np.array_equal(codes_np(codes), rc), "quantizer codes differ from the oracle"
    assert np.array_equal(scales.cpu().numpy().reshape(rs.shape), rs), "quantizer scales differ from the oracle"
    return codes, Scale(scales, kind, rpb or 0), oq.dequantize(rc, rs, out, kind, rpb)


def prepare(mode, q, k, v):
    """-> (gpu operands dict, oracle q, k, v float64)"""
    spec = MODES[mode] or {}
    g = {"q": q.to(DEV), "k": k.to(DEV), "v": v.to(DEV), "sf_q": None, "sf_k": None, "sf_v": None}
    ref = {"q": f64(q), "k": f64(k), "v": f64(v)}
    for name in ("q", "k", "v"):
        if name in spec:
            c, s, d = quantize_both({"q": q, "k": k, "v": v}[name], spec[name])
            g[name], g["sf_" + name], ref[name] = c, s, d
    return g, ref["q"], ref["k"], ref["v"]


def check(mode, o, ref, atol=Q8_ATOL):
    o = f64(o)
    if mode == "bf16":
        assert_close_bf16(o, ref)
    else:
        assert_close_q8(o, ref, atol=atol)


def run_dense(mode, B, Hq, Hkv, Sq, Skv, D, causal, seed, with_lse=False, p_terms=None, atol=Q8_ATOL):
    if mode == "fp8":
        q, k, v = workloads.outlier_qkv(seed, B, max(Sq, Skv), Hq, D)
        q, k, v = q[:, :Sq], k[:, :Skv, :Hkv], v[:, :Skv, :Hkv]
    elif mode == "sage":
        q, _, _ = workloads.biased_qk_v(seed, B, Sq, Hq, D)
        _, k, v = workloads.biased_qk_v(seed + 1, B, Skv, Hkv, D)
    else:
        q, k, v = workloads.normal_qkv(seed, B, Sq, Skv, Hq, Hkv, D)
    g, rq, rk, rv = prepare(mode, q.contiguous(), k.contiguous(), v.contiguous())
    scale = 1 / math.sqrt(D)
    lse = torch.full((B, Hq, Sq), float("nan"), device=DEV) if with_lse else None
    sf_p = None
    if mode == "sage":  # per-row-block P scale: P is stored as 224 p (lazy-rescale bound 2^1 * 224 <= 448)
        sf_p = Scale(torch.full((B, Hq, math.ceil(Sq / 128)), workloads.SAGE_SF_P, device=DEV), "per_token_block", 128)
    if p_terms is None:
        p_terms = 1
    o = fmha.fmha_fwd(g["q"], g["k"], g["v"], sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"], sf_p=sf_p,
                      softmax_scale=scale, causal=causal, lse=lse, p_terms=p_terms)
    fmha.get_device_error()
    ref_o, ref_lse = oa.attention(rq, rk, rv, scale, causal)
    check(mode, o, ref_o, atol)
    if with_lse:
        got = lse.cpu().numpy().astype(np.float64)
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(got), fin)
        # BF16 P and two-term E4M3 P: the row sum adds the unrounded exponentials;
        # one E4M3 term: it also carries E4M3 rounding (of the stored values, or of
        # each tile's largest weight), which moves lse by at most ln(1 + 2^-4)
        bound = 2e-2 if mode == "bf16" or p_terms == 2 else math.log1p(2.0 ** -4) + 2e-3
        assert np.abs(got[fin] - ref_lse[fin]).max() < bound
    return o


def test_tiny_workload():
    w = workloads.tiny()
    o = fmha.fmha_fwd(w["q"].to(DEV), w["k"].to(DEV), w["v"].to(DEV), softmax_scale=w["scale"])
    fmha.get_device_error()
    ref, _ = oa.attention(f64(w["q"]), f64(w["k"]), f64(w["v"]), w["scale"])
    assert_close_bf16(f64(o), ref)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Skv,D,causal", [
    (1, 1, 1, 1, 1, 64, False),
    (1, 2, 2, 7, 7, 128, False),
    (1, 2, 2, 129, 129, 128, True),
    (2, 4, 2, 300, 300, 128, True),     # GQA, head-paired CTAs
    (1, 2, 1, 257, 513, 64, False),     # GQA group 2, D=64
    (1, 3, 1, 200, 100, 128, True),     # Sq > Skv causal: leading rows see nothing
    (1, 1, 1, 513, 1000, 128, True),    # Sq < Skv causal (bottom-right)
    (1, 8, 8, 1024, 1024, 128, False),  # many CTAs
    (1, 4, 4, 640, 2048, 64, True),
])
def test_bf16(B, Hq, Hkv, Sq, Skv, D, causal):
    run_dense("bf16", B, Hq, Hkv, Sq, Skv, D, causal, seed=B * 1000 + Sq + Skv + D, with_lse=True)


@pytest.mark.parametrize("mode", ["pv8", "fp8", "sage"])
@pytest.mark.parametrize("Sq,Skv,causal,Hq,Hkv", [(300, 300, False, 2, 2), (1024, 1024, True, 2, 2),
                                                  (700, 1500, False, 4, 2), (129, 129, True, 1, 1)])
def test_8bit_modes(mode, Sq, Skv, causal, Hq, Hkv):
    """One E4M3 term of P (the precision every 8-bit workload states), whole heads."""
    run_dense(mode, 1, Hq, Hkv, Sq, Skv, 128, causal, seed=7 * Sq + Skv, with_lse=True)


@pytest.mark.parametrize("Sq,Skv,causal", [(2048, 2048, False), (4096, 4096, False), (4096, 4096, True)])
def test_sage_one_term_p_longer(Sq, Skv, causal):
    """One-term Sage on longer rows: its biased scores sharpen the softmax as Skv grows."""
    run_dense("sage", 1, 2, 2, Sq, Skv, 128, causal, seed=3 * Sq + 11, with_lse=True, p_terms=1)


@pytest.mark.parametrize("Sq,Skv,causal,Hq,Hkv", [(300, 300, False, 2, 2), (1024, 1024, True, 2, 2),
                                                  (700, 1500, False, 4, 2), (2048, 2048, False, 2, 2),
                                                  (2048, 2048, True, 2, 2)])
def test_sage_two_term_p(Sq, Skv, causal, Hq, Hkv):
    """Sage with P split into two E4M3 terms (the more precise option)."""
    run_dense("sage", 1, Hq, Hkv, Sq, Skv, 128, causal, seed=7 * Sq + Skv + 1, with_lse=True, p_terms=2)


def test_empty_kv_gives_zero_and_minus_inf():
    q, k, v = workloads.normal_qkv(3, 1, 200, 1, 2, 2, 128)
    lse = torch.zeros(1, 2, 200, device=DEV)
    o = fmha.fmha_fwd(q.to(DEV), k[:, :0].contiguous().to(DEV), v[:, :0].contiguous().to(DEV), lse=lse)
    fmha.get_device_error()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_output_view_is_written_in_place_only():
    q, k, v = workloads.normal_qkv(4, 1, 333, 333, 2, 2, 128)
    big = torch.full((1, 333, 5, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    view = big[:, :, 2:4, :]
    fmha.fmha_fwd(q.to(DEV), k.to(DEV), v.to(DEV), out=view)
    fmha.get_device_error()
    ref, _ = oa.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128))
    assert_close_bf16(f64(view), ref)
    assert torch.all(torch.isnan(big[:, :, :2])) and torch.all(torch.isnan(big[:, :, 4:]))


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse(mode, causal):
    B, Hq, Hkv, S, D = 2, 4, 2, 700, 128
    if mode == "bf16":
        q, k, v = workloads.normal_qkv(11, B, S, S, Hq, Hkv, D)
    else:
        q, k, v = workloads.outlier_qkv(11, B, S, Hq, D)
        k, v = k[:, :, :Hkv], v[:, :, :Hkv]
    mask = workloads.block_mask(12, B, Hkv, S, S, density=0.4)
    mask[1, 0, 3, :] = 0  # one fully hidden query block
    g, rq, rk, rv = prepare(mode, q.contiguous(), k.contiguous(), v.contiguous())
    o = fmha.fmha_fwd_block_sparse(g["q"], g["k"], g["v"], mask.to(DEV), sf_q=g["sf_q"], sf_k=g["sf_k"],
                                   sf_v=g["sf_v"], causal=causal)
    fmha.get_device_error()
    ref, _ = oa.attention(rq, rk, rv, 1 / math.sqrt(D), causal, mask.numpy())
    check(mode, o, ref)


@pytest.mark.parametrize("page_size", [16, 32, 64, 128])
def test_paged_matches_oracle_and_contiguous(page_size):
    B, Hq, Hkv, S, D = 2, 4, 2, 1000, 128
    w = workloads.sparse_paged(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D, page_size=page_size)
    mask = w["mask"]
    kp, vp, pt = w["k_pool"].to(DEV), w["v_pool"].to(DEV), w["page_table"].to(DEV)
    o = fmha.fmha_fwd_paged(w["q"].to(DEV), kp, vp, pt, S, mask=mask.to(DEV))
    fmha.get_device_error()
    kk = oa.gather_paged(f64(w["k_pool"]), w["page_table"].numpy(), S)
    vv = oa.gather_paged(f64(w["v_pool"]), w["page_table"].numpy(), S)
    ref, _ = oa.attention(f64(w["q"]), kk, vv, w["scale"], False, mask.numpy())
    assert_close_bf16(f64(o), ref)
    oc = fmha.fmha_fwd_block_sparse(w["q"].to(DEV), w["k"].to(DEV), w["v"].to(DEV), mask.to(DEV))
    assert torch.equal(o, oc), "paged and contiguous K/V must give identical bits"


def test_paged_bad_page_index_is_reported():
    w = workloads.sparse_paged(S=256, B=1, Hq=2, Hkv=2, D=128)
    pt = w["page_table"].clone()
    pt[0, 1] = 10_000
    fmha.fmha_fwd_paged(w["q"].to(DEV), w["k_pool"].to(DEV), w["v_pool"].to(DEV), pt.to(DEV), 256)
    with pytest.raises(fmha.FmhaError) as e:
        fmha.get_device_error()
    assert e.value.status == 5
    fmha.get_device_error()  # cleared


def test_invalid_arguments_raise():
    q, k, v = workloads.normal_qkv(5, 1, 64, 64, 2, 2, 128)
    with pytest.raises(fmha.FmhaError) as e:
        fmha.fmha_fwd(q.to(DEV), k[:, :, :1].to(DEV).expand(1, 64, 2, 128), v.to(DEV), causal=True)
    assert e.value.status == 1


@pytest.mark.parametrize("mode", ["pv8", "fp8"])
def test_two_term_p_is_more_accurate(mode):
    """P split into two E4M3 terms must cut the error against the oracle well below
    the one-term error and stay within the 8-bit tolerance."""
    B, Hq, Hkv, S, D = 1, 2, 2, 1024, 128
    q, k, v = workloads.normal_qkv(31, B, S, S, Hq, Hkv, D)
    g, rq, rk, rv = prepare(mode, q, k, v)
    ref, _ = oa.attention(rq, rk, rv, 1 / math.sqrt(D), True)
    errs = []
    for terms in (1, 2):
        o = fmha.fmha_fwd(g["q"], g["k"], g["v"], sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"], causal=True,
                          p_terms=terms)
        fmha.get_device_error()
        check(mode, o, ref)
        errs.append(np.abs(f64(o) - ref).max())
    assert errs[1] < errs[0] / 3, errs


def test_two_term_p_needs_8bit_v():
    q, k, v = workloads.normal_qkv(32, 1, 64, 64, 1, 1, 128)
    with pytest.raises(fmha.FmhaError) as e:
        fmha.fmha_fwd(q.to(DEV), k.to(DEV), v.to(DEV), p_terms=2)
    assert e.value.status == 1


def test_wait_limit_reports_timeout_and_context_survives():
    """A one-cycle wait limit makes the first device wait that does not succeed
    at once give up: the kernel records a timeout, lets its issued copies and
    MMAs finish, frees TMEM and returns. The host sees FMHA_ERR_TIMEOUT and the
    next launch, with the default limit, is correct."""
    q, k, v = (t.to(DEV) for t in workloads.normal_qkv(21, 1, 4096, 4096, 8, 8, 128))
    fmha.set_wait_timeout_cycles(1)
    try:
        fmha.fmha_fwd(q, k, v)
        with pytest.raises(fmha.FmhaError) as e:
            fmha.get_device_error()
        assert e.value.status == fmha.FMHA_ERR_TIMEOUT
    finally:
        fmha.set_wait_timeout_cycles(0)
    fmha.get_device_error()  # the error word was cleared by the read above
    qs, ks, vs = workloads.normal_qkv(22, 1, 300, 300, 2, 2, 128)
    o = fmha.fmha_fwd(qs.to(DEV), ks.to(DEV), vs.to(DEV))
    fmha.get_device_error()
    ref, _ = oa.attention(f64(qs), f64(ks), f64(vs), 1 / math.sqrt(128))
    assert_close_bf16(f64(o), ref)
