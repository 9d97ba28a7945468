"""Full-size parity: every workload at its full size, in the launch
configuration bench.py times (GPU quantizer -> attention), checked on sampled
outputs the oracle computes row by row.

For a few sampled (batch, head) pairs the oracle quantizes that head's
operands itself (per-tensor scales use the oracle's amax over the whole
tensor), the GPU codes of those heads must match bit for bit, and sampled
query rows (first, boundary, last and random rows) must match the oracle's
float64 attention within the path's tolerance. The first sampled head of
every workload is checked whole: every row and column element by element,
and the cosine similarity over the whole head.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import e4m3 as oe
from oracle import quant as oq
from precision_attention_fmha_b200 import fmha, workloads
from precision_attention_fmha_b200.fmha import Scale
from tests.helpers import BF16_ATOL, Q8_ATOL, Q8_COS, codes_np, cos_per_head, f32, f64

pytestmark = [pytest.mark.gpu, pytest.mark.big]
DEV = torch.device("cuda")
TDT = {"int8": torch.int8, "e4m3": torch.float8_e4m3fn}


def sample_rows(S, n_random=8, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2, 127, 128, S // 2, S - 2, S - 1]
    return np.unique(np.clip(np.concatenate([fixed, rng.integers(0, S, n_random)]), 0, S - 1))


def oracle_head(x_bf16, b, h, spec, full_x=None):
    """Oracle dequantized operand of one (b, h) slice [S, D] (float64), plus its codes.
    spec None = BF16 operand used as is."""
    xs = f32(x_bf16[b:b + 1, :, h:h + 1, :])
    if spec is None:
        return xs[0, :, 0].astype(np.float64), None
    out, kind, rpb = spec
    if kind == "per_tensor":  # the scale comes from the whole tensor's amax
        scale = oq.scale_from_amax(np.max(np.abs(f32(full_x))), out)
        codes = oq.codes_with_scale(xs, scale, out)
        deq = oq.dequantize(codes, np.array([scale]), out, "per_tensor")
    else:
        codes, sc = oq.quantize_blockwise(xs, out, kind, rpb)
        deq = oq.dequantize(codes, sc, out, kind, rpb)
    return deq[0, :, 0], codes[0, :, 0]


def check_rows(mode, got_rows, ref_rows, sf_o=None, atol=Q8_ATOL):
    """got/ref: dict (b, h) -> [n, D] arrays. sf_o: the output scale of an E4M3
    output, whose rounding (2^-4 relative, 2^-10 sf_o absolute) adds to the
    8-bit tolerance; the per-head cosine bound stays Q8_COS (measured 1 - cos
    about 7e-4 for the E4M3-output workload)."""
    for key in ref_rows:
        g, r = got_rows[key], ref_rows[key]
        assert np.all(np.isfinite(g)), f"non-finite output at {key}"
        if sf_o is not None:
            bound = 2.0 ** -4 * np.abs(r) + 2.0 ** -10 * sf_o + Q8_ATOL * max(1.0, np.abs(r).max())
            worst = np.argmax(np.abs(g - r) - bound)
            assert np.all(np.abs(g - r) <= bound), f"{key}: err {np.abs(g - r).flat[worst]:.3e}"
            c = cos_per_head(g[None, :, None, :], r[None, :, None, :])[0]
            assert c >= Q8_COS, f"{key}: cos {c:.6f}"
            continue
        err = np.abs(g - r).max()
        if mode == "bf16":
            assert err <= BF16_ATOL, f"{key}: max-abs {err:.3e}"
        else:
            scale = max(1.0, np.abs(r).max())
            assert err <= atol * scale, f"{key}: max-abs {err:.3e} > {atol} x {scale:.2f}"
            c = cos_per_head(g[None, :, None, :], r[None, :, None, :])[0]
            assert c >= Q8_COS, f"{key}: cos {c:.6f}"


def whole_or_rows(q_head, rows, k_head, v_head, scale, Sq, causal, block_mask_bh=None):
    """Oracle output for query rows `rows` of one head: the whole head through the
    chunked attention, a sample through the row-wise one."""
    if len(rows) == Sq:
        bm = None if block_mask_bh is None else block_mask_bh[None, None]
        o, _ = oa.attention(q_head[None, :, None, :], k_head[None, :, None, :], v_head[None, :, None, :], scale,
                            causal, bm)
        return o[0, :, 0, :]
    o, _ = oa.attention_rows(q_head[rows], rows, k_head, v_head, scale, Sq, causal, block_mask_bh)
    return o


def run_case(mode, q, k, v, specs, heads, causal=False, sf_p=None, p_terms=1, o8=False, atol=Q8_ATOL):
    """Quantize on the GPU exactly as bench.py does, run attention, compare sampled rows.
    o8: E4M3 output with V's per-tensor scale as sf_o (bench.py's E4M3-output workload)."""
    B, Sq, Hq, D = q.shape
    Skv = k.shape[1]
    group = Hq // k.shape[2]
    ops, sfs = {"q": q.to(DEV), "k": k.to(DEV), "v": v.to(DEV)}, {}
    host = {"q": q, "k": k, "v": v}
    for name, spec in specs.items():
        out, kind, rpb = spec
        c, sc = fmha.fmha_quantize_blockwise(ops[name], TDT[out], kind, rpb)
        ops[name], sfs["sf_" + name] = c, Scale(sc, kind, rpb or 0)
    extra, sf_o = {}, None
    if o8:
        extra = {"out": torch.empty((B, Sq, Hq, v.shape[3]), dtype=torch.float8_e4m3fn, device=DEV),
                 "sf_o": sfs["sf_v"]}
        sf_o = float(sfs["sf_v"].tensor.reshape(-1)[0].item())
    o = fmha.fmha_fwd(ops["q"], ops["k"], ops["v"], softmax_scale=1 / math.sqrt(D), causal=causal, sf_p=sf_p,
                      p_terms=p_terms, **sfs, **extra)
    fmha.get_device_error()
    got, ref = {}, {}
    for (b, h) in heads:
        hk = h // group
        opr = {}
        for name, hh in (("q", h), ("k", hk), ("v", hk)):
            spec = specs.get(name)
            deq, codes = oracle_head(host[name], b, hh, spec, host[name] if spec and spec[1] == "per_tensor" else None)
            if codes is not None:  # GPU codes of this head must equal the oracle's
                gc = codes_np(ops[name][b:b + 1, :, hh:hh + 1, :].contiguous())[0, :, 0]
                assert np.array_equal(gc, codes), f"{name} codes differ for head ({b}, {hh})"
            opr[name] = deq
        # the first sampled head whole, the others on sampled rows
        rows = np.arange(Sq) if (b, h) == heads[0] else sample_rows(Sq, seed=b * 131 + h)
        ro = whole_or_rows(opr["q"], rows, opr["k"], opr["v"], 1 / math.sqrt(D), Sq, causal)
        ref[(b, h)] = ro
        if o8:
            got[(b, h)] = oe.decode(o.view(torch.uint8)[b, rows, h, :].cpu().numpy()) * sf_o
        else:
            got[(b, h)] = f64(o[b, rows, h, :])
    check_rows(mode, got, ref, sf_o, atol)


@pytest.mark.parametrize("S", [4096, 16384, 32768])
def test_dense_pv8_full_size(S):
    w = workloads.dense_pv8(S=S)
    run_case("pv8", w["q"], w["k"], w["v"], {"v": ("e4m3", "per_tensor", None)}, heads=[(0, 0), (0, 17), (0, 39)])


def test_dense_pv8_e4m3_output_full_size():
    w = workloads.dense_pv8(S=32768)
    run_case("pv8", w["q"], w["k"], w["v"], {"v": ("e4m3", "per_tensor", None)}, heads=[(0, 0), (0, 39)], o8=True)


@pytest.mark.parametrize("causal", [False, True])
def test_all_fp8_full_size(causal):
    w = workloads.all_fp8()
    spec = {n: ("e4m3", "per_head", None) for n in "qkv"}
    run_case("fp8", w["q"], w["k"], w["v"], spec, heads=[(0, 0), (1, 13), (1, 31)], causal=causal)


@pytest.mark.parametrize("p_terms", [1, 2])
def test_sage_full_size(p_terms):
    """The Sage workload as stated (one E4M3 term of P with a per-row-block scale) and
    with P split into two E4M3 terms."""
    w = workloads.sage()
    B, S, H, D = w["q"].shape
    spec = {"q": ("int8", "per_token_block", 128), "k": ("int8", "per_token_block", 64),
            "v": ("e4m3", "per_channel", None)}
    sf_p = Scale(torch.full((B, H, math.ceil(S / 128)), workloads.SAGE_SF_P, device=DEV), "per_token_block", 128)
    run_case("sage", w["q"], w["k"], w["v"], spec, heads=[(0, 0), (0, 11), (0, 23)], sf_p=sf_p, p_terms=p_terms)


@pytest.mark.parametrize("mode", ["bf16", "pv8", "fp8"])
def test_wide_qk_full_size(mode):
    """D_qk = 192 / D_v = 128, B1 H40 S16384, quantized as bench.py's wide_qk workloads."""
    w = workloads.wide_qk(outliers=mode == "fp8")
    spec = {"bf16": {}, "pv8": {"v": ("e4m3", "per_tensor", None)},
            "fp8": {n: ("e4m3", "per_head", None) for n in "qkv"}}[mode]
    run_case(mode, w["q"], w["k"], w["v"], spec, heads=[(0, 0), (0, 19), (0, 39)])


def test_sparse_paged_full_size():
    """The paged block-sparse workload against the oracle, and its contiguous-K/V
    control (bench.py's sparse_contig workload) equal to it bit for bit."""
    w = workloads.sparse_paged()
    B, S, Hq, D = w["q"].shape
    Hkv = w["k"].shape[2]
    group = Hq // Hkv
    q, dmask = w["q"].to(DEV), w["mask"].to(DEV)
    o = fmha.fmha_fwd_paged(q, w["k_pool"].to(DEV), w["v_pool"].to(DEV), w["page_table"].to(DEV), S,
                            mask=dmask, softmax_scale=w["scale"])
    fmha.get_device_error()
    oc = fmha.fmha_fwd_block_sparse(q, w["k"].to(DEV), w["v"].to(DEV), dmask, softmax_scale=w["scale"])
    fmha.get_device_error()
    assert torch.equal(o, oc), "paged and contiguous K/V must give identical bits"
    del oc
    mask = w["mask"].numpy()
    got, ref = {}, {}
    heads = [(0, 0), (1, 21), (3, 63)]
    for (b, h) in heads:
        hk = h // group
        kk = oa.gather_paged(f64(w["k_pool"][:, :, hk:hk + 1]), w["page_table"].numpy()[b:b + 1], S)[0, :, 0]
        vv = oa.gather_paged(f64(w["v_pool"][:, :, hk:hk + 1]), w["page_table"].numpy()[b:b + 1], S)[0, :, 0]
        rows = np.arange(S) if (b, h) == heads[0] else sample_rows(S, seed=b * 7 + h)
        ro = whole_or_rows(f64(w["q"][b, :, h, :]), rows, kk, vv, w["scale"], S, False, mask[b, hk])
        ref[(b, h)] = ro
        got[(b, h)] = f64(o[b, rows, h, :])
    check_rows("bf16", got, ref)


def test_decode_paged_full_size():
    """The decode workload (Sq = 1, B4 Hq64 Hkv8 Skv16384, 64-token pages, 25 % of the
    128-key blocks kept) with automatic splits, as bench.py launches it: every output
    row and its LSE against the oracle (the whole output is 256 rows)."""
    from tests.helpers import assert_close_bf16

    w = workloads.decode_paged()
    B, Sq, Hq, D = w["q"].shape
    S = w["k"].shape[1]
    lse = torch.full((B, Hq, Sq), float("nan"), device=DEV)
    o = fmha.fmha_fwd_decode(w["q"].to(DEV), w["k_pool"].to(DEV), w["v_pool"].to(DEV),
                             page_table=w["page_table"].to(DEV), Skv=S, mask=w["mask"].to(DEV),
                             softmax_scale=w["scale"], lse=lse)
    fmha.get_device_error()
    ref, ref_lse = oa.attention(f64(w["q"]), f64(w["k"]), f64(w["v"]), w["scale"], False, w["mask"].numpy())
    assert_close_bf16(f64(o), ref)
    got = f64(lse)
    assert np.all(np.isfinite(got)) and np.abs(got - ref_lse).max() < 2e-2
