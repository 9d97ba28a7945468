"""Seeded synthetic inputs for the five attention workloads.

This module only draws random tensors with the shapes, distributions and
structure of the workloads; it holds none of the attention or quantization
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it. Random draws use numpy's PCG64 (``default_rng(seed)``) in float32,
then round to BF16 (round-to-nearest-even, via torch's CPU cast); the very
same BF16 bytes go to the GPU and to the oracle.

Workloads (B, heads, sequence lengths, head dim, distributions):

* ``tiny``        B=1 H=1 Sq=Skv=256 D=64, BF16 N(0,1), scale 1/sqrt(64).
* ``dense_pv8``   B=1 H=40 D=128 Sq=Skv in {4096, 16384, 32768}; Q, K BF16
                  N(0,1); V N(0,1) to be quantized per tensor to E4M3.
* ``all_fp8``     B=2 H=32 D=128 Sq=Skv=8192; Q, K, V N(0,1) where each entry
                  independently (prob. 0.01) is multiplied by 20 (outliers);
                  quantized per head to E4M3.
* ``sage``        B=1 H=24 D=128 Sq=Skv=16384; Q and K are N(0,1) plus a
                  per-(head, channel) bias drawn from N(0, 2) (variance 2),
                  separately for Q and K and shared over tokens; V N(0,1).
* ``sparse_paged`` B=4 Hq=64 Hkv=8 D=128 Sq=Skv=16384, BF16 N(0,1); K/V in a
                  pool of 64-token pages addressed through a seeded random
                  page-table permutation; 128x128 block mask per (b, kv head)
                  drawn Bernoulli(0.25) with the diagonal block forced on.
* ``wide_qk``     the dense workload with a 192-wide Q/K head dim and a
                  128-wide V: B=1 H=40 Sq=Skv=16384, BF16 N(0,1) (with the
                  all_fp8 outliers when ``outliers``), scale 1/sqrt(192).

Every generator takes the sizes as arguments so tests can draw small cases
with the same recipe.
"""

import math

import numpy as np
import torch

SEED_BASE = 1000


def _normal_bf16(rng, shape):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def normal_qkv(seed, B, Sq, Skv, Hq, Hkv, D):
    """Q [B,Sq,Hq,D], K/V [B,Skv,Hkv,D] in BF16, N(0,1)."""
    rng = np.random.default_rng(seed)
    return _normal_bf16(rng, (B, Sq, Hq, D)), _normal_bf16(rng, (B, Skv, Hkv, D)), _normal_bf16(rng, (B, Skv, Hkv, D))


def outlier_qkv(seed, B, S, H, D, p=0.01, factor=20.0):
    """N(0,1) with iid Bernoulli(p) entries multiplied by ``factor``, BF16."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        x = rng.standard_normal(size=(B, S, H, D), dtype=np.float32)
        hit = rng.random(size=x.shape, dtype=np.float32) < p
        x = np.where(hit, x * np.float32(factor), x)
        out.append(torch.from_numpy(x).to(torch.bfloat16))
    return tuple(out)


def biased_qk_v(seed, B, S, H, D, bias_var=2.0):
    """Q, K = N(0,1) + bias[h, d] with bias ~ N(0, bias_var) (one draw for Q, one
    for K, shared over batch and tokens); V = N(0,1). All BF16."""
    rng = np.random.default_rng(seed)
    std = np.float32(math.sqrt(bias_var))
    qb = rng.standard_normal(size=(H, D), dtype=np.float32) * std
    kb = rng.standard_normal(size=(H, D), dtype=np.float32) * std
    q = rng.standard_normal(size=(B, S, H, D), dtype=np.float32) + qb
    k = rng.standard_normal(size=(B, S, H, D), dtype=np.float32) + kb
    v = rng.standard_normal(size=(B, S, H, D), dtype=np.float32)
    return tuple(torch.from_numpy(x).to(torch.bfloat16) for x in (q, k, v))


def block_mask(seed, B, Hkv, Sq, Skv, density=0.25, block=128):
    """uint8 [B, Hkv, ceil(Sq/block), ceil(Skv/block)], Bernoulli(density), diagonal forced on."""
    rng = np.random.default_rng(seed)
    nq, nk = -(-Sq // block), -(-Skv // block)
    m = (rng.random(size=(B, Hkv, nq, nk)) < density).astype(np.uint8)
    d = np.arange(min(nq, nk))
    m[:, :, d, d] = 1
    return torch.from_numpy(m)


def paged_pool(seed, k, v, page_size=64, extra_pages=0):
    """Scatter contiguous K/V [B,S,H,D] into a pool of pages through a seeded
    random permutation. Returns (k_pool [P,page,H,D], v_pool [P,page,H,Dv],
    page_table int32 [B, pages_per_seq]). Unused pool pages (``extra_pages``)
    hold N(0,1) noise."""
    B, S, H, D = k.shape
    per_seq = -(-S // page_size)
    P = B * per_seq + extra_pages
    rng = np.random.default_rng(seed)
    perm = rng.permutation(P)[: B * per_seq].reshape(B, per_seq).astype(np.int32)
    kp = _normal_bf16(rng, (P, page_size, H, D))
    vp = _normal_bf16(rng, (P, page_size, H, v.shape[3]))
    for b in range(B):
        for i in range(per_seq):
            t0, t1 = i * page_size, min(S, (i + 1) * page_size)
            kp[perm[b, i], : t1 - t0] = k[b, t0:t1]
            vp[perm[b, i], : t1 - t0] = v[b, t0:t1]
    return kp, vp, torch.from_numpy(perm)


# ---- the five named workloads (full sizes; tests pass smaller sizes) ----

def tiny(S=256, D=64, B=1, H=1):
    q, k, v = normal_qkv(SEED_BASE + 1, B, S, S, H, H, D)
    return dict(q=q, k=k, v=v, scale=1.0 / math.sqrt(D))


def dense_pv8(S=16384, B=1, H=40, D=128):
    q, k, v = normal_qkv(SEED_BASE + 2 + S, B, S, S, H, H, D)
    return dict(q=q, k=k, v=v, scale=1.0 / math.sqrt(D))


def all_fp8(S=8192, B=2, H=32, D=128):
    q, k, v = outlier_qkv(SEED_BASE + 3 + S, B, S, H, D)
    return dict(q=q, k=k, v=v, scale=1.0 / math.sqrt(D))


def wide_qk(S=16384, B=1, H=40, D=192, Dv=128, outliers=False):
    """Q, K [B,S,H,D] and V [B,S,H,Dv] (D != Dv): N(0,1), or with 1% x20 outliers."""
    seed = SEED_BASE + 6 + S
    if outliers:
        q, k, _ = outlier_qkv(seed, B, S, H, D)
        _, _, v = outlier_qkv(seed + 1, B, S, H, Dv)
    else:
        q, k, _ = normal_qkv(seed, B, S, S, H, H, D)
        _, _, v = normal_qkv(seed + 1, B, S, S, H, H, Dv)
    return dict(q=q, k=k, v=v, scale=1.0 / math.sqrt(D))


# P scale of the Sage workload's one-term E4M3 P, per 128-row query block: P is
# stored as 224 p. With the lazy-rescale threshold it implies (tau = 1: the row
# max may grow by 2x before O is rescaled) a stored P stays <= 448, and small
# weights keep 3.8 more binades above E4M3's subnormal range than with 1/16.
SAGE_SF_P = 1.0 / 224


def sage(S=16384, B=1, H=24, D=128):
    q, k, v = biased_qk_v(SEED_BASE + 4 + S, B, S, H, D)
    return dict(q=q, k=k, v=v, scale=1.0 / math.sqrt(D))


def sparse_paged(S=16384, B=4, Hq=64, Hkv=8, D=128, page_size=64, density=0.25):
    seed = SEED_BASE + 5 + S
    q, k, v = normal_qkv(seed, B, S, S, Hq, Hkv, D)
    kp, vp, pt = paged_pool(seed + 1, k, v, page_size)
    mask = block_mask(seed + 2, B, Hkv, S, S, density)
    return dict(q=q, k=k, v=v, k_pool=kp, v_pool=vp, page_table=pt, mask=mask,
                page_size=page_size, scale=1.0 / math.sqrt(D))


def decode_mask(seed, B, Hkv, Sq, Skv, density=0.25, block=128):
    """Block mask for decode shapes: Bernoulli(density) over KV blocks, the last
    KV block (the newest tokens) always kept."""
    rng = np.random.default_rng(seed)
    nq, nk = -(-Sq // block), -(-Skv // block)
    m = (rng.random(size=(B, Hkv, nq, nk)) < density).astype(np.uint8)
    m[:, :, :, nk - 1] = 1
    return torch.from_numpy(m)


def decode_paged(S=16384, B=4, Hq=64, Hkv=8, D=128, Sq=1, page_size=64, density=0.25):
    """Decode step over a block-sparse paged cache: Sq query tokens per sequence
    against S cached tokens (GQA Hq/Hkv), pages in a seeded permutation."""
    seed = SEED_BASE + 6 + S
    q, _, _ = normal_qkv(seed, B, Sq, 1, Hq, Hkv, D)
    _, k, v = normal_qkv(seed + 1, B, 1, S, Hq, Hkv, D)
    kp, vp, pt = paged_pool(seed + 2, k, v, page_size)
    mask = decode_mask(seed + 3, B, Hkv, Sq, S, density)
    return dict(q=q, k=k, v=v, k_pool=kp, v_pool=vp, page_table=pt, mask=mask,
                page_size=page_size, scale=1.0 / math.sqrt(D))
