"""Scaled-dot-product attention in float64 (the definition the FMHA computes).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name the operation -- "Dense Context FMHA" over QK (BMM1), softmax,
PV (BMM2) ("FlashInfer FP8/BF16 mixed-precision attention for Blackwell",
introduction and section 1; "FlashInfer DiT optimization: SageAttention and
Int8/FP8 mixed-precision kernels", section 2) -- but never write it down. The
textbook definition is used, on dequantized operands:

    s_ij = softmax_scale * <q_i, k_j>          (masked pairs: -inf)
    p_ij = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)
    o_i  = sum_j p_ij v_j
    lse_i = max_j s_ij + log sum_j exp(s_ij - max_j s_ij)

Readings where the pages are silent:

* Layout: token-major [B, S, H, D]; GQA maps query head h to KV head
  h // (Hq // Hkv) (the "GQA 64/8" workload of "FlashInfer block-sparse
  attention with PrimTS", "Why" item 1).
* Causal with Sq != Skv is bottom-right aligned: key j is visible to query i
  iff j <= i + (Skv - Sq).
* The block mask is 128 x 128 in logical token coordinates, one byte per
  (b, kv_head, q_block, kv_block); it is ANDed with the causal mask.
* A row with no visible key has o = 0 and lse = -inf.
* Paged K/V ("FlashInfer block-sparse attention with PrimTS", section 2: a
  page table maps each sequence's logical pages to pool pages) is the same
  attention on the gathered sequence: ``gather_paged``.

Rows are processed in chunks of 512 with a float64 matmul; nothing else is
blocked, fused or reordered.
"""

import numpy as np

BLOCK = 128
ROW_CHUNK = 512


def visible_mask(Sq, Skv, causal, block_mask_bh=None, block=BLOCK):
    """Boolean [Sq, Skv]: which keys each query sees (for one (b, kv head))."""
    vis = np.ones((Sq, Skv), dtype=bool)
    if causal:
        i = np.arange(Sq)[:, None]
        j = np.arange(Skv)[None, :]
        vis &= j <= i + (Skv - Sq)
    if block_mask_bh is not None:
        bm = np.asarray(block_mask_bh).astype(bool)
        rows = np.arange(Sq) // block
        cols = np.arange(Skv) // block
        vis &= bm[rows[:, None], cols[None, :]]
    return vis


def attention(q, k, v, softmax_scale, causal=False, block_mask=None, block=BLOCK):
    """q [B, Sq, Hq, D], k/v [B, Skv, Hkv, D] (any real dtype, used in float64).

    block_mask: None or array [B, Hkv, ceil(Sq/block), ceil(Skv/block)] (nonzero = keep).
    Returns (o [B, Sq, Hq, D] float64, lse [B, Hq, Sq] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, Dv = v.shape
    assert k.shape[:3] == (B, Skv, Hkv) and k.shape[3] == D and Hq % Hkv == 0
    group = Hq // Hkv
    o = np.zeros((B, Sq, Hq, Dv), dtype=np.float64)
    lse = np.full((B, Hq, Sq), -np.inf, dtype=np.float64)
    for b in range(B):
        for hk in range(Hkv):
            bm = None if block_mask is None else block_mask[b, hk]
            vis_full = visible_mask(Sq, Skv, causal, bm, block)
            kk = k[b, :, hk, :]  # [Skv, D]
            vv = v[b, :, hk, :]
            for g in range(group):
                h = hk * group + g
                for r0 in range(0, Sq, ROW_CHUNK):
                    r1 = min(Sq, r0 + ROW_CHUNK)
                    s = softmax_scale * np.matmul(q[b, r0:r1, h, :], kk.T)  # [rows, Skv]
                    vis = vis_full[r0:r1]
                    s = np.where(vis, s, -np.inf)
                    m = np.max(s, axis=1, keepdims=True) if Skv else np.full((r1 - r0, 1), -np.inf)
                    alive = np.isfinite(m)
                    m_safe = np.where(alive, m, 0.0)
                    e = np.exp(s - m_safe)  # exp(-inf) = 0 for masked keys
                    l = np.sum(e, axis=1, keepdims=True)
                    p = np.divide(e, l, out=np.zeros_like(e), where=l > 0)
                    o[b, r0:r1, h, :] = np.matmul(p, vv)
                    lse[b, h, r0:r1] = np.where(alive[:, 0], m[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)), -np.inf)
    return o, lse


def gather_paged(pool, page_table, Skv):
    """Paged K or V pool [num_pages, page_size, H, D] + page_table [B, max_pages]
    -> the logical sequence [B, Skv, H, D]: token t of sequence b is row
    t % page_size of pool page page_table[b, t // page_size]."""
    pool = np.asarray(pool)
    pt = np.asarray(page_table)
    page_size = pool.shape[1]
    t = np.arange(Skv)
    pages = pt[:, t // page_size]  # [B, Skv]
    return pool[pages, (t % page_size)[None, :]]  # [B, Skv, H, D]


def probabilities(q, k, softmax_scale, causal=False, block_mask_bh=None, block=BLOCK):
    """P = softmax rows for one (b, h) pair: q [Sq, D], k [Skv, D] -> [Sq, Skv].

    Used by the invariant tests (rows sum to one, masked entries are zero).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    s = softmax_scale * (q @ k.T)
    vis = visible_mask(q.shape[0], k.shape[0], causal, block_mask_bh, block)
    s = np.where(vis, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return np.divide(e, l, out=np.zeros_like(e), where=l > 0)


def attention_rows(q_rows, rows, k, v, softmax_scale, Sq, causal=False, block_mask_bh=None, block=BLOCK):
    """The same attention for selected query rows of one (batch, KV head).

    q_rows [n, D] are the queries at absolute positions ``rows`` (of Sq); k, v
    [Skv, D] are that KV head's keys and values; block_mask_bh is its
    [ceil(Sq/block), ceil(Skv/block)] block mask or None. Returns
    (o [n, D], lse [n]) in float64 -- for spot checks of full-size outputs.
    """
    q = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    rows = np.asarray(rows)
    Skv = k.shape[0]
    s = softmax_scale * (q @ k.T)
    j = np.arange(Skv)[None, :]
    vis = np.ones(s.shape, dtype=bool)
    if causal:
        vis &= j <= rows[:, None] + (Skv - Sq)
    if block_mask_bh is not None:
        bm = np.asarray(block_mask_bh).astype(bool)
        vis &= bm[(rows // block)[:, None], (np.arange(Skv) // block)[None, :]]
    s = np.where(vis, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    alive = np.isfinite(m)
    m_safe = np.where(alive, m, 0.0)
    e = np.exp(s - m_safe)
    l = np.sum(e, axis=1, keepdims=True)
    p = np.divide(e, l, out=np.zeros_like(e), where=l > 0)
    lse = np.where(alive[:, 0], m[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)), -np.inf)
    return p @ v, lse
