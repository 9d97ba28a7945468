"""Decode path (GQA-packed query tiles, split-KV, split merge) against the oracle.

fmha_fwd_decode computes the same attention as fmha_fwd / fmha_fwd_paged
("FlashInfer block-sparse attention with PrimTS", section 1: the query tile
is the query block times the query heads per KV head); the oracle is the same
float64 attention, so the bars are those of the dense path. With one split the
result must equal fmha_fwd bit for bit: every row sees the same operands in
the same order, only its TMEM lane differs (when all rows fit one tile the
CTA's two query tiles split the KV tiles, so there are always two partials).
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from precision_attention_fmha_b200 import fmha, workloads
from tests.helpers import f64
from tests.test_fmha_gpu import check, prepare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def to_pool(x, page_table, page_size):
    """Scatter x [B, S, H, D] (any dtype) into pool pages by page_table [B, pages]."""
    B, S, H, D = x.shape
    xb = x.view(torch.uint8) if x.element_size() == 1 else x
    pool = torch.zeros((int(page_table.max()) + 1, page_size, H, D), dtype=xb.dtype)
    for b in range(B):
        for i in range(page_table.shape[1]):
            t0, t1 = i * page_size, min(S, (i + 1) * page_size)
            if t0 < S:
                pool[int(page_table[b, i]), : t1 - t0] = xb[b, t0:t1]
    return pool.view(x.dtype) if x.element_size() == 1 else pool


def decode_case(mode, B, Hq, Hkv, Sq, Skv, splits, causal, paged, masked, seed):
    q, _, _ = workloads.normal_qkv(seed, B, Sq, 1, Hq, Hkv, 128)
    _, k, v = workloads.normal_qkv(seed + 1, B, 1, Skv, Hq, Hkv, 128)
    g, rq, rk, rv = prepare(mode, q, k, v)
    mask = workloads.decode_mask(seed + 2, B, Hkv, Sq, Skv, 0.5) if masked else None
    lse = torch.full((B, Hq, Sq), float("nan"), device=DEV)
    kw = dict(sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"], causal=causal, lse=lse, num_splits=splits,
              mask=mask.to(DEV) if masked else None)
    if paged:  # pool the GPU operands (codes for 8-bit) page by page; the oracle keeps contiguous K/V
        _, _, pt = workloads.paged_pool(seed + 3, k, v, 64)
        kp, vp = to_pool(g["k"].cpu(), pt, 64), to_pool(g["v"].cpu(), pt, 64)
        o = fmha.fmha_fwd_decode(g["q"], kp.to(DEV), vp.to(DEV), page_table=pt.to(DEV), Skv=Skv, **kw)
    else:
        o = fmha.fmha_fwd_decode(g["q"], g["k"], g["v"], **kw)
    fmha.get_device_error()
    ref, ref_lse = oa.attention(rq, rk, rv, 1 / math.sqrt(128), causal, mask.numpy() if masked else None)
    check(mode, o, ref)
    got_lse = f64(lse)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got_lse), fin)
    tol = 2e-2 if mode == "bf16" else math.log1p(2 ** -4) + 2e-3
    assert np.abs(got_lse[fin] - ref_lse[fin]).max() <= tol
    return g, o, kw


@pytest.mark.parametrize("mode,B,Hq,Hkv,Sq,Skv,splits,causal,paged,masked", [
    ("bf16", 2, 16, 2, 1, 2000, 0, False, True, True),     # decode, G = 8, automatic splits, paged + mask
    ("bf16", 2, 16, 2, 1, 2000, 1, False, True, False),    # one split, two interleaved partials
    ("bf16", 1, 8, 1, 5, 1000, 3, True, False, False),     # causal, contiguous, ragged token tail
    ("bf16", 2, 32, 2, 40, 1500, 4, True, True, False),    # G = 16, 640 packed rows = 3 unit pairs
    ("bf16", 1, 4, 4, 33, 900, 2, False, False, True),     # G = 1 (MHA)
    ("bf16", 1, 128, 1, 2, 600, 2, False, False, False),   # G = 128: one token per unit
    ("bf16", 1, 8, 1, 1, 300, 8, False, False, False),     # more splits asked than KV tiles
    # at most 16 packed rows: the 16-lane softmax pass, both row halves
    ("bf16", 2, 32, 2, 1, 1500, 0, False, True, True),     # G = 16, one token: rows 0-15
    ("bf16", 1, 8, 1, 2, 1000, 2, True, False, False),     # G = 8, two tokens, causal
    ("bf16", 1, 4, 1, 3, 700, 0, True, False, True),      # G = 4, three tokens: rows 0-11
    ("pv8", 2, 16, 2, 4, 2000, 0, True, True, False),
    ("fp8", 2, 16, 2, 1, 3000, 5, False, True, True),
    ("fp8", 1, 8, 2, 9, 1200, 3, True, False, False),
])
def test_decode_matches_oracle(mode, B, Hq, Hkv, Sq, Skv, splits, causal, paged, masked):
    decode_case(mode, B, Hq, Hkv, Sq, Skv, splits, causal, paged, masked, seed=Sq * 101 + Skv + Hq)


@pytest.mark.parametrize("mode", ["bf16", "fp8"])
def test_one_split_equals_dense_bits(mode):
    # 40 tokens x 8 heads = 320 packed rows: more than one 128-row tile, so one
    # split means one partial per row and the packed TMA store writes O directly.
    B, Hq, Hkv, Sq, Skv = 2, 16, 2, 40, 1000
    q, _, _ = workloads.normal_qkv(41, B, Sq, 1, Hq, Hkv, 128)
    _, k, v = workloads.normal_qkv(42, B, 1, Skv, Hq, Hkv, 128)
    g, _, _, _ = prepare(mode, q, k, v)
    kw = dict(sf_q=g["sf_q"], sf_k=g["sf_k"], sf_v=g["sf_v"], causal=True)
    o1 = fmha.fmha_fwd_decode(g["q"], g["k"], g["v"], num_splits=1, **kw)
    o2 = fmha.fmha_fwd(g["q"], g["k"], g["v"], **kw)
    fmha.get_device_error()
    assert torch.equal(o1, o2)


def test_fully_hidden_rows_give_zero_and_minus_inf():
    B, Hq, Hkv, Sq, Skv = 2, 8, 2, 2, 700
    q, _, _ = workloads.normal_qkv(51, B, Sq, 1, Hq, Hkv, 128)
    _, k, v = workloads.normal_qkv(52, B, 1, Skv, Hq, Hkv, 128)
    mask = torch.ones((B, Hkv, 1, 6), dtype=torch.uint8)
    mask[1, 0] = 0  # batch 1, KV head 0: nothing visible
    lse = torch.zeros((B, Hq, Sq), device=DEV)
    o = fmha.fmha_fwd_decode(q.to(DEV), k.to(DEV), v.to(DEV), mask=mask.to(DEV), num_splits=3, lse=lse)
    fmha.get_device_error()
    assert torch.all(o[1, :, :4] == 0) and torch.all(torch.isneginf(lse[1, :4]))
    ref, _ = oa.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128), False, mask.numpy())
    check("bf16", o, ref)


def test_decode_argument_errors():
    q, _, _ = workloads.normal_qkv(61, 1, 1, 1, 6, 2, 128)
    _, k, v = workloads.normal_qkv(62, 1, 1, 512, 6, 2, 128)
    with pytest.raises(fmha.FmhaError) as e:  # group of 3 heads: not a power of two
        fmha.fmha_fwd_decode(q.to(DEV), k.to(DEV), v.to(DEV))
    assert e.value.status == fmha.FMHA_ERR_UNSUPPORTED
    q, _, _ = workloads.normal_qkv(63, 1, 1, 1, 8, 2, 128)
    _, k, v = workloads.normal_qkv(64, 1, 1, 2048, 8, 2, 128)
    small = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(fmha.FmhaError) as e:  # workspace too small for 4 splits
        fmha.fmha_fwd_decode(q.to(DEV), k.to(DEV), v.to(DEV), num_splits=4, workspace=small)
    assert e.value.status == fmha.FMHA_ERR_INVALID_ARG
    assert fmha.decode_num_splits(q, k, num_splits=4) == 4
    assert fmha.decode_num_splits(q, k, num_splits=100) == 16  # at most one split per KV tile
