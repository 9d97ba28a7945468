"""Pins for oracle/online_softmax.py (the tiled online softmax with P rounded to
BF16 or E4M3), on the CPU.

Pinned against: the exact attention of oracle/attention.py (itself pinned to
brute force and torch) when P is kept unrounded, at every rescale threshold and
tile size; the threshold's closed form; a single visible key, whose weight the
row-sum correction makes exact; the stale-max bound 2^tau * g <= 448; and error
bounds derived from the formats' rounding (E4M3: 2^-4 relative, two E4M3 terms:
2^-7, BF16: 2^-8), computed from the exact softmax probabilities alone.
"""

import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import online_softmax as OS


def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("tau", [0.0, 1.0, 8.0])
@pytest.mark.parametrize("tile", [16, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_unrounded_online_pass_equals_exact_attention(tau, tile, causal):
    """Scores spread over many binades, so the lazy max moves (or not) at every
    threshold; GQA, Sq != Skv, a block mask with a hidden block."""
    rng = np.random.default_rng(31)
    B, Sq, Skv, Hq, Hkv, D, Dv, blk = 2, 150, 230, 4, 2, 8, 6, 32
    q, k, v = _rand(rng, B, Sq, Hq, D) * 2, _rand(rng, B, Skv, Hkv, D) * 2, _rand(rng, B, Skv, Hkv, Dv)
    bm = rng.random((B, Hkv, -(-Sq // blk), -(-Skv // blk))) < 0.7
    bm[0, 1, 2, :] = False  # one fully hidden query block
    stats = {}
    o, lse = OS.attention_rounded_p(q, k, v, 0.9, causal, bm, p_mode="exact", block=blk, tile=tile, tau=tau,
                                    stats=stats)
    ref, ref_lse = A.attention(q, k, v, 0.9, causal, bm, blk)
    assert np.allclose(o, ref, atol=1e-12, rtol=0)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin) and np.allclose(lse[fin], ref_lse[fin], atol=1e-12)
    if tau < 8.0:
        assert stats["rescales"] > 0  # the rescale path ran


@pytest.mark.parametrize("sf_p,tau", [(1 / 224, 1.0), (1 / 16, 4.0), (1 / 448, 0.0), (1.0, 8.0), (1e-3, 0.0),
                                      (1 / 28, 4.0), (1 / 27.9, 4.0)])
def test_threshold_closed_form(sf_p, tau):
    """tau = floor(log2(448 sf_p)) clamped to [0, 8]: the largest tau with 2^tau / sf_p <= 448."""
    assert OS.tau_for("e4m3", sf_p) == tau
    assert OS.tau_for("bf16", sf_p) == 8.0
    assert 2.0 ** tau / sf_p <= 448.0 * (1 + 1e-12) or tau == 0.0


@pytest.mark.parametrize("p_mode", ["e4m3", "e4m3x2", "bf16"])
def test_single_visible_key_returns_its_value_exactly(p_mode):
    """Each row sees one key: its stored weight E4M3(g) = 192 for g = 200 (a tie,
    to even) differs from p = 200, and only the row-sum correction (one term)
    or the low term (two terms) brings O back to v (to the last bit of the
    float64 division). The one-term LSE is the log of the corrected sum, so it
    sits ln(192 / 200) below the exact score."""
    rng = np.random.default_rng(32)
    S, D = 40, 8
    q, k, v = _rand(rng, 1, S, 1, D), _rand(rng, 1, S, 1, D), _rand(rng, 1, S, 1, D)
    bm = np.eye(S, dtype=bool)[None, None]  # block size 1: key i for query i only
    o, lse = OS.attention_rounded_p(q, k, v, 0.5, False, bm, p_mode=p_mode, sf_p=1 / 200, block=1)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=1e-15, atol=0)
    s = 0.5 * np.einsum("sd,sd->s", q[0, :, 0], k[0, :, 0])
    shift = math.log(192.0 / 200.0) if p_mode == "e4m3" else 0.0
    assert np.allclose(lse[0, 0], s + shift, atol=1e-12, rtol=0)


def test_stale_max_stays_within_e4m3_range():
    """Tile maxima rising by 0.9 log2 units (below tau = 1) move no max, so
    stored P climbs above g = 224 (to E4M3(2^0.9 * 224) = 416) and never past
    448; a rise of 1.1 moves the max instead."""
    D = 4
    for rise, rescales, top in ((0.9, 0, 416.0), (1.1, 2, 224.0)):
        k = np.zeros((1, 3 * 128, 1, D))
        for t in range(3):
            k[0, t * 128, 0, 0] = min(t, 1) * rise  # key 0 of tile t scores min(t, 1) * rise in log2 units
        k[0, 2 * 128, 0, 0] = 2 * rise if rise > 1 else rise
        q = np.zeros((1, 1, 1, D))
        q[0, 0, 0, 0] = 1.0
        v = np.ones((1, 3 * 128, 1, D))
        stats = {}
        o, _ = OS.attention_rounded_p(q, k, v, math.log(2.0), p_mode="e4m3", sf_p=1 / 224, stats=stats)
        assert stats["rescales"] == rescales and stats["max_stored"] == top and stats["max_stored"] <= 448.0
        assert np.allclose(o, 1.0, atol=2 ** -4)


def _bound_terms(q, k, v, scale, causal, tile=128):
    """Exact softmax probabilities p, sum_j p_j |v_j| and sum over tiles of the tile's largest p."""
    p = A.probabilities(q[0, :, 0], k[0, :, 0], scale, causal)
    spv = p @ np.abs(v[0, :, 0])
    pmax = sum(p[:, c0:c0 + tile].max(axis=1) for c0 in range(0, p.shape[1], tile))
    return p, spv, pmax


@pytest.mark.parametrize("causal", [False, True])
def test_one_e4m3_term_within_its_rounding_bound(causal):
    """Every stored weight is normal and unsaturated (|s2| <= 16 * 0.2 * log2(e)
    < 4.7, so 224 * 2^-10.4 < p <= 448 with tau = 1), so E4M3 moves it by at
    most 2^-4 of itself (plus the float32 rounding of p):
    |O_p - O| <= 2^-4 (sum_j p_j |v_j| + |O| sum_t pmax_t) / (1 - 2^-4 sum_t pmax_t)."""
    rng = np.random.default_rng(33)
    S, D = 600, 16
    q = rng.uniform(-1, 1, (1, S, 1, D))
    k = rng.uniform(-1, 1, (1, S, 1, D))
    v = _rand(rng, 1, S, 1, D)
    scale = 0.2  # |s2| <= 16 * 0.2 * log2(e) < 5
    o, lse = OS.attention_rounded_p(q, k, v, scale, causal, p_mode="e4m3", sf_p=1 / 224)
    ref, ref_lse = A.attention(q, k, v, scale, causal)
    _, spv, pmax = _bound_terms(q, k, v, scale, causal)
    r = ref[0, :, 0]
    bound = 2.0 ** -4 * (spv + np.abs(r) * pmax[:, None]) / (1 - 2.0 ** -4 * pmax[:, None])
    err = np.abs(o[0, :, 0] - r)
    assert np.all(err <= bound * (1 + 1e-6) + 1e-9)
    assert err.max() > 1e-3  # the rounding is really there
    assert np.all(np.abs(lse - ref_lse) <= -np.log1p(-(2.0 ** -4) * pmax)[None] + 1e-12)


@pytest.mark.parametrize("p_mode,rel", [("e4m3x2", 2.0 ** -7), ("bf16", 2.0 ** -8)])
def test_finer_p_within_its_rounding_bound(p_mode, rel):
    """Two E4M3 terms (hi + lo, the residual through f16) and BF16 P: the row sum
    is the unrounded one, so |O_p - O| <= rel * sum_j p_j |v_j|."""
    rng = np.random.default_rng(34)
    S, D = 600, 16
    q = rng.uniform(-1, 1, (1, S, 1, D))
    k = rng.uniform(-1, 1, (1, S, 1, D))
    v = _rand(rng, 1, S, 1, D)
    o, lse = OS.attention_rounded_p(q, k, v, 0.2, True, p_mode=p_mode, sf_p=1 / 224)
    ref, ref_lse = A.attention(q, k, v, 0.2, True)
    _, spv, _ = _bound_terms(q, k, v, 0.2, True)
    err = np.abs(o[0, :, 0] - ref[0, :, 0])
    assert np.all(err <= rel * spv * (1 + 1e-6) + 1e-9)
    assert err.max() > rel * 1e-3
    assert np.allclose(lse, ref_lse, atol=1e-6)


def test_two_terms_beat_one():
    rng = np.random.default_rng(35)
    q, k, v = _rand(rng, 1, 300, 2, 16), _rand(rng, 1, 400, 1, 16), _rand(rng, 1, 400, 1, 8)
    ref, _ = A.attention(q, k, v, 0.5, False)
    e1 = np.abs(OS.attention_rounded_p(q, k, v, 0.5, p_mode="e4m3", sf_p=1 / 224)[0] - ref).max()
    e2 = np.abs(OS.attention_rounded_p(q, k, v, 0.5, p_mode="e4m3x2", sf_p=1 / 224)[0] - ref).max()
    assert e2 < e1 / 8


def test_per_block_p_scales_apply_to_their_rows():
    """A scale array [B, Hq, ceil(Sq / 128)] gives each 128-row block its own
    g and tau: the result equals running each block alone with its scale."""
    rng = np.random.default_rng(36)
    q, k, v = _rand(rng, 1, 300, 1, 8), _rand(rng, 1, 260, 1, 8), _rand(rng, 1, 260, 1, 8)
    sfp = np.array([[[1 / 224, 1 / 16, 1 / 448]]])
    o, lse = OS.attention_rounded_p(q, k, v, 0.7, True, p_mode="e4m3", sf_p=sfp)
    for i, s in enumerate(sfp[0, 0]):
        r0, r1 = 128 * i, min(300, 128 * (i + 1))
        oi, li = OS.attention_rounded_p(q, k, v, 0.7, True, p_mode="e4m3", sf_p=s)
        assert np.array_equal(o[:, r0:r1], oi[:, r0:r1]) and np.array_equal(lse[:, :, r0:r1], li[:, :, r0:r1])


def test_bf16_rounding_matches_an_independent_encoder():
    """BF16 P rounding (round to nearest, ties to even) against ml_dtypes, on
    random float32 values and on every tie between two neighbouring BF16 values
    of a few binades."""
    import ml_dtypes

    rng = np.random.default_rng(37)
    x = np.concatenate([rng.uniform(0, 300, 100000), rng.standard_normal(100000)]).astype(np.float32)
    hi16 = (np.arange(0x3F00, 0x4400, dtype=np.uint32) << 16).view(np.float32)
    ties = ((hi16.view(np.uint32) | 0x8000).view(np.float32))  # halfway to the next BF16 value
    x = np.concatenate([x, ties, hi16])
    want = x.astype(ml_dtypes.bfloat16).astype(np.float32)
    assert np.array_equal(OS._round_bf16(x), want)


def test_sage_p_scale_reading():
    """The Sage workload's P scale: on its operands (biased INT8 Q/K in 128- and
    64-token blocks, E4M3 V per channel), one E4M3 term of P stored as 224 p
    (sf_p = 1/224, tau = 1) is closer to the exact attention than one stored as
    16 p (sf_p = 2^-4, tau = 4): the small weights sit 3.8 binades further from
    E4M3's subnormal range. Two terms are closer still."""
    import torch

    from oracle import quant as Q
    from precision_attention_fmha_b200 import workloads

    q, k, v = (t.to(torch.float32).numpy() for t in workloads.biased_qk_v(5, 1, 1024, 2, 128))
    qd = Q.dequantize(*Q.quantize_blockwise(q, "int8", "per_token_block", 128), "int8", "per_token_block", 128)
    kd = Q.dequantize(*Q.quantize_blockwise(k, "int8", "per_token_block", 64), "int8", "per_token_block", 64)
    vd = Q.dequantize(*Q.quantize_blockwise(v, "e4m3", "per_channel"), "e4m3", "per_channel")
    scale = 1 / math.sqrt(128)
    ref, _ = A.attention(qd, kd, vd, scale)
    err = {(mode, sfp): np.abs(OS.attention_rounded_p(qd, kd, vd, scale, p_mode=mode, sf_p=sfp)[0] - ref).max()
           for mode in ("e4m3", "e4m3x2") for sfp in (1 / 16, 1 / 224)}
    assert err[("e4m3", 1 / 224)] < err[("e4m3", 1 / 16)]
    assert err[("e4m3x2", 1 / 224)] < err[("e4m3", 1 / 224)] / 8


@pytest.mark.parametrize("causal", [False, True])
def test_split_states_merge_to_the_exact_attention(causal):
    """Two running states over alternate kept tiles, merged with the
    2^(m_x - M) weights: with P unrounded the merge is the exact attention,
    whatever the thresholds (causal with Skv > Sq, a block mask with a hidden
    query block, GQA)."""
    rng = np.random.default_rng(38)
    B, Sq, Skv, Hq, Hkv, D, Dv = 1, 300, 700, 2, 1, 8, 6
    q, k, v = _rand(rng, B, Sq, Hq, D) * 2, _rand(rng, B, Skv, Hkv, D) * 2, _rand(rng, B, Skv, Hkv, Dv)
    bm = rng.random((B, Hkv, 3, 6)) < 0.6
    bm[0, 0, 1, :] = False
    bm[0, 0, 2, :] = [True, False, True, True, False, True]
    ref, ref_lse = A.attention(q, k, v, 0.9, causal, bm)
    for tau in (0.0, 8.0):
        o, lse = OS.attention_rounded_p(q, k, v, 0.9, causal, bm, p_mode="exact", tau=tau, split_kv=True)
        assert np.allclose(o, ref, atol=1e-12, rtol=0)
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(lse), fin) and np.allclose(lse[fin], ref_lse[fin], atol=1e-12)


def test_split_dealing_and_kept_tiles():
    """The tiles a query tile keeps (its last row's causal bound, the block mask)
    and their dealing by rank parity."""
    assert OS._kept_tiles(0, 0, 0, 300, 700, True, None, 128) == [0, 128, 256, 384, 512]  # last row 527
    assert OS._kept_tiles(0, 0, 2, 300, 700, True, None, 128) == [0, 128, 256, 384, 512, 640]
    assert OS._kept_tiles(0, 0, 0, 700, 300, True, None, 128) == []  # rows 0..127 see no key (bottom-right)
    bm = np.zeros((1, 1, 3, 6), dtype=bool)
    bm[0, 0, 1, [0, 2, 3, 5]] = True
    assert OS._kept_tiles(0, 0, 1, 300, 700, False, bm, 128) == [0, 256, 384, 640]
    assert OS._deal([0, 256, 384, 640, 768]) == ([0, 384, 768], [256, 640])


@pytest.mark.parametrize("p_mode,rel", [("e4m3", None), ("bf16", 2.0 ** -8)])
def test_split_states_within_the_rounding_bounds(p_mode, rel):
    """The rounded modes through two states stay within the same format bounds
    (each state's row sum carries its own tiles' corrections)."""
    rng = np.random.default_rng(39)
    S, D = 600, 16
    q = rng.uniform(-1, 1, (1, S, 1, D))
    k = rng.uniform(-1, 1, (1, S, 1, D))
    v = _rand(rng, 1, S, 1, D)
    o, _ = OS.attention_rounded_p(q, k, v, 0.2, True, p_mode=p_mode, sf_p=1 / 224, split_kv=True)
    ref, _ = A.attention(q, k, v, 0.2, True)
    _, spv, pmax = _bound_terms(q, k, v, 0.2, True)
    r = ref[0, :, 0]
    if rel is None:
        bound = 2.0 ** -4 * (spv + np.abs(r) * pmax[:, None]) / (1 - 2.0 ** -4 * pmax[:, None])
    else:
        bound = rel * spv
    assert np.all(np.abs(o[0, :, 0] - r) <= bound * (1 + 1e-6) + 1e-9)


@pytest.mark.parametrize("B,Sq,Hq,Hkv,Skv,causal,masked", [
    (2, 1, 16, 2, 2000, False, True),   # one token, G = 8: all rows in one tile (two partials per split)
    (1, 5, 8, 1, 1000, True, False),    # causal, ragged token tail
    (2, 40, 32, 2, 1500, True, False),  # G = 16: 640 packed rows, five tiles
    (1, 33, 4, 4, 900, False, True),    # G = 1
    (1, 2, 128, 1, 600, False, False),  # G = 128: one token per tile
    (1, 130, 2, 1, 700, True, True),    # tiles across a 128-token mask row
])
@pytest.mark.parametrize("n_splits", [1, 3, 8])
def test_decode_schedule_merges_to_the_exact_attention(B, Sq, Hq, Hkv, Skv, causal, masked, n_splits):
    """Packed rows, ranked and split KV tiles, interleaved partials and the
    log-sum-exp merge: with P unrounded, the exact attention."""
    rng = np.random.default_rng(40 + Sq + n_splits)
    q, k, v = _rand(rng, B, Sq, Hq, 128) * 2, _rand(rng, B, Skv, Hkv, 128) * 2, _rand(rng, B, Skv, Hkv, 128)
    bm = None
    if masked:
        bm = rng.random((B, Hkv, -(-Sq // 128), -(-Skv // 128))) < 0.5
        bm[..., -1] = True
    ref, ref_lse = A.attention(q, k, v, 0.1, causal, bm)
    o, lse = OS.decode_rounded_p(q, k, v, 0.1, causal, bm, p_mode="exact", n_splits=n_splits)
    assert np.allclose(o, ref, atol=1e-12, rtol=0)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin) and np.allclose(lse[fin], ref_lse[fin], atol=1e-12)


def test_decode_split_groups():
    kept = list(range(7))
    assert OS._split_groups(kept, 3, False) == [[0, 1, 2], [3, 4, 5], [6]]
    assert OS._split_groups(kept, 3, True) == [[0, 2], [1], [3, 5], [4], [6], []]
    assert OS._split_groups(kept, 8, False) == [[0], [1], [2], [3], [4], [5], [6], []]
    assert OS._split_groups([], 2, True) == [[], [], [], []]


@pytest.mark.parametrize("p_mode,rel", [("e4m3", None), ("bf16", 2.0 ** -8)])
def test_decode_schedule_within_the_rounding_bounds(p_mode, rel):
    """The partials' merge weights are their row sums, so the rounded decode
    schedule keeps the single-pass bounds (one token, G = 8, three splits)."""
    rng = np.random.default_rng(41)
    Skv, D = 2000, 16
    q = rng.uniform(-1, 1, (1, 1, 8, D))
    k = rng.uniform(-1, 1, (1, Skv, 1, D))
    v = _rand(rng, 1, Skv, 1, D)
    o, _ = OS.decode_rounded_p(q, k, v, 0.2, False, None, p_mode=p_mode, sf_p=1 / 224, n_splits=3)
    ref, _ = A.attention(q, k, v, 0.2, False)
    for h in range(8):
        qh = q[:, :, h:h + 1]
        _, spv, pmax = _bound_terms(qh, k, v, 0.2, False)
        r = ref[0, :, h]
        if rel is None:
            bound = 2.0 ** -4 * (spv + np.abs(r) * pmax[:, None]) / (1 - 2.0 ** -4 * pmax[:, None])
        else:
            bound = rel * spv
        assert np.all(np.abs(o[0, :, h] - r) <= bound * (1 + 1e-6) + 1e-9)
