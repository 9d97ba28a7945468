"""Attention through the tiled online softmax with P rounded as the kernels store it.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

``attention.attention`` is the exact definition on dequantized operands. This
module takes the steps of the method that approximate it, in the pages' order:
the scores of one query row are taken 128 keys at a time; the running row max
moves lazily, only when a tile's max exceeds it by more than tau (log2 units),
and then O and the row sum are rescaled ("FlashInfer FP8/BF16 mixed-precision
attention for Blackwell", section 3, with tau = 8 there); P is cast to BF16, or
to E4M3 after multiplication by g = 1 / sf_p, the P scale factor of
"FlashInfer DiT optimization: SageAttention and Int8/FP8 mixed-precision
kernels", section 2; O accumulates P V; the epilogue divides by the row sum.

Readings where the pages are silent (the same the kernels take):

* Scores are in log2 units: s2 = softmax_scale * log2(e) * <q, k>.
* The first tile in which a row sees a key sets its max; later tiles move it
  (with O and l scaled by 2^(m_old - m_new)) only when their max exceeds it
  by more than tau.
* p = 2^(s2 - m) * g is formed in float32 (here: exactly, then rounded once
  to float32; the "exact" mode keeps it in float64), so a stale max gives
  p <= 2^tau * g.
* tau = 8 for BF16 P; for E4M3 P, tau = floor(log2(448 * sf_p)) clamped to
  [0, 8], so 2^tau * g <= 448. sf_p is one value, or one per (b, h_q,
  128-row query block); without one, sf_p = 2^-4.
* BF16 P: stored = RN_bf16(p); the row sum adds the unrounded p.
* One E4M3 term: stored = E4M3(p) (RN-even, saturating); the row sum adds
  the unrounded p plus, per tile, E4M3(p_max) - p_max for the tile's largest
  p (so a dominant key's weight is normalised by its stored value).
* Two E4M3 terms: hi = E4M3(p), lo = E4M3(RN_f16(RN_f16(p) - hi)), stored =
  hi + lo; the row sum adds the unrounded p.
* O = (sum over tiles of stored P V) / l; lse = (m + log2(l / g)) * ln 2;
  a row with no visible key has O = 0 and lse = -inf.

Not modelled: the exp2 unit's own error (here 2^x is exact before the float32
rounding), and the order of the float32 additions of the row sum (here float64).
These move a stored code only where p sits on an E4M3 or BF16 rounding
boundary. The D_qk = 192 kernels with one query tile per CTA split the KV tiles
of a row between two running states and merge them at the end; this module
follows the single-state pass.
"""

import math

import numpy as np

from . import e4m3
from .attention import visible_mask

TILE = 128
LOG2E = 1.0 / math.log(2.0)


def _round_bf16(x32):
    """float32 array -> nearest BF16 value (ties to even), as float32."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _round_e4m3(x):
    return e4m3.decode(e4m3.encode(x))


def _round_f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def tau_for(p_mode, sf_p):
    """Lazy-rescale threshold in log2 units for one P scale."""
    if p_mode == "bf16":
        return 8.0
    return float(min(8.0, max(0.0, math.floor(math.log2(448.0 * sf_p)))))


def _tile_pass(s2, vv, tiles, tile, p_mode, g, tau, counters):
    """One running state over the KV tiles ``tiles`` (start columns, in order)
    for the rows of s2 [rows, Skv] (log2 scores, -inf where hidden); vv [Skv, Dv].
    Returns (acc [rows, Dv], l [rows], m [rows]): O before normalisation, the
    row sum and the lazy max."""
    n, Dv = s2.shape[0], vv.shape[1]
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    acc = np.zeros((n, Dv))
    for c0 in tiles:
        c1 = min(s2.shape[1], c0 + tile)
        st = s2[:, c0:c1]
        m_tile = st.max(axis=1)
        seen = np.isfinite(m_tile)
        first = seen & ~np.isfinite(m)
        move = seen & np.isfinite(m) & (m_tile > m + tau)
        alpha = np.exp2(np.where(move, m - np.where(move, m_tile, 0.0), 0.0))
        acc *= alpha[:, None]
        l *= alpha
        counters["rescales"] += int(move.sum())
        m = np.where(first | move, m_tile, m)
        m_use = np.where(np.isfinite(m), m, 0.0)
        p = np.exp2(st - m_use[:, None]) * g  # 0 where hidden
        if p_mode != "exact":  # the kernels form p in float32
            p = p.astype(np.float32).astype(np.float64)
        if p_mode == "exact":
            stored, corr = p, 0.0
        elif p_mode == "bf16":
            stored, corr = _round_bf16(p).astype(np.float64), 0.0
        elif p_mode == "e4m3":
            stored = _round_e4m3(p)
            pmax = np.where(seen, (np.exp2(np.where(seen, m_tile - m_use, 0.0)) * g), 0.0)
            pmax = pmax.astype(np.float32).astype(np.float64)
            corr = np.where(seen, _round_e4m3(pmax) - pmax, 0.0)
        elif p_mode == "e4m3x2":
            hi = _round_e4m3(p)
            lo = _round_e4m3(_round_f16(_round_f16(p) - hi))
            stored, corr = hi + lo, 0.0
        else:
            raise ValueError(p_mode)
        if stored.size:
            counters["max_stored"] = max(counters["max_stored"], float(stored.max()))
        l += p.sum(axis=1) + corr
        acc += stored @ vv[c0:c1]
    return acc, l, m


def _kept_tiles(b, hk, qblk, Sq, Skv, causal, block_mask, tile):
    """Start columns of the KV tiles a 128-row query tile keeps: within its
    causal bound (its last row's) and kept by the block mask, in order."""
    n = -(-Skv // tile)
    if causal:
        last = min(qblk * tile + tile - 1, Sq - 1) + (Skv - Sq)
        n = 0 if last < 0 else min(n, last // tile + 1)
    return [u * tile for u in range(n) if block_mask is None or block_mask[b, hk, qblk, u]]


def _deal(kept):
    """Kept tiles by rank: even ranks to the first state, odd to the second."""
    return kept[0::2], kept[1::2]


def attention_rounded_p(q, k, v, softmax_scale, causal=False, block_mask=None, p_mode="e4m3", sf_p=None,
                        p_block=128, block=128, tile=TILE, tau=None, split_kv=False, stats=None):
    """q [B, Sq, Hq, D], k [B, Skv, Hkv, D], v [B, Skv, Hkv, Dv] (dequantized values).

    p_mode: "bf16", "e4m3" (one term), "e4m3x2" (two terms) or "exact" (P kept
    unrounded: the online pass alone, which must equal ``attention.attention``).
    sf_p: None (2^-4 for the E4M3 modes), a number, or an array [B, Hq,
    ceil(Sq / p_block)] of per-query-block scales. tau: None (the reading's
    threshold) or a number (the "exact" mode's rescale logic can then be
    exercised at any threshold). split_kv: the kept KV tiles of each 128-row
    query tile are dealt by rank to two running states (even ranks to one, odd
    to the other), which are merged at the end:
    O = (acc_0 2^(m_0 - M) + acc_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)),
    M = max(m_0, m_1) (the one-query-tile schedule of the 192-wide QK kernels;
    needs 128-key tiles, 128-row P blocks and a 128 x 128 block mask).
    stats: optional dict that receives the largest stored P and the number of
    rescales. Returns (o [B, Sq, Hq, Dv] float64, lse [B, Hq, Sq] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, Dv = v.shape
    group = Hq // Hkv
    if split_kv and not (tile == p_block == block == TILE):
        raise ValueError("split_kv follows the kernels' 128-row, 128-key tiles")
    if sf_p is None:
        sf_p = 2.0 ** -4
    sfp_arr = np.asarray(sf_p, dtype=np.float64)
    o = np.zeros((B, Sq, Hq, Dv))
    lse = np.full((B, Hq, Sq), -np.inf)
    counters = {"max_stored": 0.0, "rescales": 0}
    for b in range(B):
        for h in range(Hq):
            hk = h // group
            bm = None if block_mask is None else block_mask[b, hk]
            vis = visible_mask(Sq, Skv, causal, bm, block)
            s2 = (softmax_scale * LOG2E) * (q[b, :, h, :] @ k[b, :, hk, :].T)
            s2 = np.where(vis, s2, -np.inf)
            vv = v[b, :, hk, :]
            for r0 in range(0, Sq, p_block):  # rows of one P-scale block
                r1 = min(Sq, r0 + p_block)
                sfp = float(sfp_arr) if sfp_arr.ndim == 0 else float(sfp_arr[b, h, r0 // p_block])
                g = 1.0 if p_mode in ("bf16", "exact") else 1.0 / sfp
                tau_r = (tau_for(p_mode, sfp) if p_mode != "exact" else 8.0) if tau is None else float(tau)
                if not split_kv:
                    acc, l, m = _tile_pass(s2[r0:r1], vv, range(0, Skv, tile), tile, p_mode, g, tau_r, counters)
                else:
                    kept = _kept_tiles(b, hk, r0 // tile, Sq, Skv, causal, block_mask, tile)
                    parts = [_tile_pass(s2[r0:r1], vv, half, tile, p_mode, g, tau_r, counters)
                             for half in _deal(kept)]
                    ms = np.stack([np.where(pl > 0, pm, -np.inf) for _, pl, pm in parts])
                    m = ms.max(axis=0)
                    m_use = np.where(np.isfinite(m), m, 0.0)
                    w = [np.where(pl > 0, np.exp2(np.where(pl > 0, pm - m_use, 0.0)), 0.0) for _, pl, pm in parts]
                    acc = parts[0][0] * w[0][:, None] + parts[1][0] * w[1][:, None]
                    l = parts[0][1] * w[0] + parts[1][1] * w[1]
                alive = l > 0
                o[b, r0:r1, h, :] = np.where(alive[:, None], acc / np.where(alive, l, 1.0)[:, None], 0.0)
                lse[b, h, r0:r1] = np.where(alive, (m + np.log2(np.where(alive, l, 1.0) / g)) * math.log(2.0),
                                            -np.inf)
    if stats is not None:
        stats.update(counters)
    return o, lse


def _split_groups(kept, n_splits, interleave):
    """The KV tile groups of a decode tile's partials: split s takes the ranks
    [s * per, (s + 1) * per) of the kept tiles, per = ceil(total / n_splits);
    with interleave, two partials per split take the split's ranks alternately
    (rank - s * per even, then odd)."""
    total = len(kept)
    per = -(-total // n_splits) if total else 0
    groups = []
    for s in range(n_splits):
        mine = kept[s * per:min(total, (s + 1) * per)]
        groups += [mine[0::2], mine[1::2]] if interleave else [mine]
    return groups


def decode_rounded_p(q, k, v, softmax_scale, causal=False, block_mask=None, p_mode="e4m3", sf_p=None, n_splits=1,
                     tile=TILE, stats=None):
    """The decode path's schedule with rounded P, for q [B, Sq, Hq, D] (a few
    query tokens), k [B, Skv, Hkv, D], v [B, Skv, Hkv, Dv].

    The Sq * G rows of one KV head (G = Hq / Hkv, a power of two) are packed
    token-major, row r = (token r // G, head r % G), into 128-row tiles (the
    query tile is the query block times the query heads per KV head, "FlashInfer
    block-sparse attention with PrimTS", section 1). Each tile ranks the KV
    tiles it keeps (its last token's causal bound, the block mask row of its
    tokens); split s of n_splits takes ranks [s * per, (s + 1) * per), per =
    ceil(total / n_splits). When all rows fit one tile, each split has two
    partials taking its ranks alternately. Every partial is one running state
    (the tiled pass with rounded P); the partials merge by their log-sum-exp:
    lse = log sum_j exp(lse_j), O = sum_j exp(lse_j - lse) O_j, O_j = acc_j / l_j.
    sf_p: None (2^-4 for the E4M3 modes) or one number. Returns (o, lse) as
    ``attention_rounded_p`` does.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, Dv = v.shape
    G = Hq // Hkv
    sfp = 2.0 ** -4 if sf_p is None else float(sf_p)
    g = 1.0 if p_mode in ("bf16", "exact") else 1.0 / sfp
    tau = tau_for(p_mode, sfp) if p_mode != "exact" else 8.0
    n_rows = Sq * G
    units = -(-n_rows // TILE)
    interleave = units == 1
    toks = TILE // G  # query tokens per 128-row tile
    n_kv = -(-Skv // tile)
    o = np.zeros((B, Sq, Hq, Dv))
    lse = np.full((B, Hq, Sq), -np.inf)
    counters = {"max_stored": 0.0, "rescales": 0}
    for b in range(B):
        for hk in range(Hkv):
            bm = None if block_mask is None else block_mask[b, hk]
            vis = visible_mask(Sq, Skv, causal, bm, TILE)  # per token
            vv = v[b, :, hk, :]
            for u in range(units):
                rows = np.arange(u * TILE, min(n_rows, (u + 1) * TILE))
                tok, head = rows // G, hk * G + rows % G
                s2 = (softmax_scale * LOG2E) * np.einsum("rd,kd->rk", q[b, tok, head, :], k[b, :, hk, :])
                s2 = np.where(vis[tok], s2, -np.inf)
                tok0 = u * toks
                n = n_kv
                if causal:
                    last = min(tok0 + toks - 1, Sq - 1) + (Skv - Sq)
                    n = 0 if last < 0 else min(n_kv, last // tile + 1)
                kept = [c * tile for c in range(n) if bm is None or bm[tok0 // TILE, c]]
                parts = [_tile_pass(s2, vv, grp, tile, p_mode, g, tau, counters)
                         for grp in _split_groups(kept, n_splits, interleave)]
                # each partial: O_j = acc / l, lse_j; then the log-sum-exp merge
                lse_j = np.stack([np.where(pl > 0, (pm + np.log2(np.where(pl > 0, pl, 1.0) / g)) * math.log(2.0),
                                           -np.inf) for _, pl, pm in parts])
                o_j = np.stack([np.where((pl > 0)[:, None], pa / np.where(pl > 0, pl, 1.0)[:, None], 0.0)
                                for pa, pl, _ in parts])
                mx = lse_j.max(axis=0)
                alive = np.isfinite(mx)
                w = np.where(np.isfinite(lse_j), np.exp(lse_j - np.where(alive, mx, 0.0)[None]), 0.0)
                wsum = w.sum(axis=0)
                o[b, tok, head, :] = np.where(alive[:, None], (w[:, :, None] * o_j).sum(axis=0)
                                              / np.where(alive, wsum, 1.0)[:, None], 0.0)
                lse[b, head, tok] = np.where(alive, np.where(alive, mx, 0.0) + np.log(np.where(alive, wsum, 1.0)),
                                             -np.inf)
    if stats is not None:
        stats.update(counters)
    return o, lse
