"""GPU attention with a 192-wide QK head dim and a 128-wide V / O head dim
(the shape "FlashInfer FP8/BF16 mixed-precision attention for Blackwell" names
in its reviewer notes as the one its shared-memory-P schedule leaves out),
against the float64 oracle, element by element.

Modes: BF16 Q/K/V, BF16 Q/K with E4M3 V (one E4M3 term of P), and all-E4M3.
With BF16 Q/K one query tile runs per CTA; with E4M3 Q/K two, each 192-byte
row copied as two 128-byte swizzle columns whose second half TMA zero-fills.
Sizes span several tiles with ragged tails, causal in both Sq / Skv orders,
GQA, paged K/V (bit-identical to contiguous) and a block mask."""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from precision_attention_fmha_b200 import fmha, workloads
from tests.helpers import assert_close_bf16, assert_close_q8, f64
from tests.test_fmha_gpu import prepare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
D, DV = 192, 128


def operands(mode, seed, B, Sq, Skv, Hq, Hkv):
    """Q/K with D = 192 and V with Dv = 128, from the workload generators."""
    if mode == "fp8":
        q, k, _ = workloads.outlier_qkv(seed, B, max(Sq, Skv), Hq, D)
        _, _, v = workloads.outlier_qkv(seed + 1, B, max(Sq, Skv), Hq, DV)
        return q[:, :Sq].contiguous(), k[:, :Skv, :Hkv].contiguous(), v[:, :Skv, :Hkv].contiguous()
    q, k, _ = workloads.normal_qkv(seed, B, Sq, Skv, Hq, Hkv, D)
    _, _, v = workloads.normal_qkv(seed + 1, B, Sq, Skv, Hq, Hkv, DV)
    return q, k, v


def check(mode, o, ref):
    assert o.shape[-1] == DV
    if mode == "bf16":
        assert_close_bf16(f64(o), ref)
    else:
        assert_close_q8(f64(o), ref)


@pytest.mark.parametrize("mode", ["bf16", "pv8", "fp8"])
@pytest.mark.parametrize("B,Hq,Hkv,Sq,Skv,causal", [
    (1, 1, 1, 1, 1, False),
    (1, 2, 2, 300, 300, False),
    (1, 2, 2, 1024, 1024, True),
    (2, 4, 2, 700, 1500, False),   # GQA, Sq < Skv
    (1, 3, 1, 200, 100, True),     # Sq > Skv causal: leading rows see nothing
    (1, 1, 1, 513, 1000, True),    # Sq < Skv causal (bottom-right)
])
def test_d192_dense(mode, B, Hq, Hkv, Sq, Skv, causal):
    q, k, v = operands(mode, 17 * Sq + Skv + B, B, Sq, Skv, Hq, Hkv)
    g, rq, rk, rv = prepare(mode, q, k, v)
    scale = 1 / math.sqrt(D)
    lse = torch.full((B, Hq, Sq), float("nan"), device=DEV)
    o = fmha.fmha_fwd(g["q"], g["k"], g["v"], sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"],
                      softmax_scale=scale, causal=causal, lse=lse)
    fmha.get_device_error()
    ref_o, ref_lse = oa.attention(rq, rk, rv, scale, causal)
    check(mode, o, ref_o)
    got = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got), fin)
    # BF16 P: unrounded row sums; one E4M3 term: within ln(1 + 2^-4) of the exact sum
    bound = 2e-2 if mode == "bf16" else math.log1p(2.0 ** -4) + 2e-3
    assert np.abs(got[fin] - ref_lse[fin]).max() < bound


@pytest.mark.parametrize("mode", ["bf16", "pv8", "fp8"])
@pytest.mark.parametrize("causal", [False, True])
def test_d192_block_sparse(mode, causal):
    B, Hq, Hkv, S = 2, 4, 2, 700
    q, k, v = operands(mode, 23, B, S, S, Hq, Hkv)
    mask = workloads.block_mask(24, B, Hkv, S, S, density=0.4)
    mask[1, 0, 3, :] = 0  # one fully hidden query block
    g, rq, rk, rv = prepare(mode, q, k, v)
    o = fmha.fmha_fwd_block_sparse(g["q"], g["k"], g["v"], mask.to(DEV), sf_q=g["sf_q"], sf_k=g["sf_k"],
                                   sf_v=g["sf_v"], causal=causal)
    fmha.get_device_error()
    ref, _ = oa.attention(rq, rk, rv, 1 / math.sqrt(D), causal, mask.numpy())
    check(mode, o, ref)


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
@pytest.mark.parametrize("page_size", [16, 64])
def test_d192_paged_matches_oracle_and_contiguous(mode, page_size):
    B, Hq, Hkv, S = 2, 4, 2, 1000
    q, k, v = operands(mode, 31 + page_size, B, S, S, Hq, Hkv)
    g, rq, rk, rv = prepare(mode, q, k, v)
    mask = workloads.block_mask(32, B, Hkv, S, S, density=0.5)
    # page the operands the kernel reads (E4M3 codes are exact in BF16 and back)
    bf = torch.bfloat16
    kp, vp, pt = workloads.paged_pool(33, g["k"].cpu().to(bf), g["v"].cpu().to(bf), page_size=page_size,
                                      extra_pages=3)
    kp, vp = kp.to(g["k"].dtype), vp.to(g["v"].dtype)  # noise pages (never read) round to E4M3
    o = fmha.fmha_fwd_paged(g["q"], kp.to(DEV), vp.to(DEV), pt.to(DEV), S, mask=mask.to(DEV), sf_q=g["sf_q"],
                            sf_k=g["sf_k"], sf_v=g["sf_v"])
    fmha.get_device_error()
    ref, _ = oa.attention(rq, rk, rv, 1 / math.sqrt(D), False, mask.numpy())
    check(mode, o, ref)
    oc = fmha.fmha_fwd_block_sparse(g["q"], g["k"], g["v"], mask.to(DEV), sf_q=g["sf_q"], sf_k=g["sf_k"],
                                    sf_v=g["sf_v"])
    assert torch.equal(o, oc), "paged and contiguous K/V must give identical bits"
