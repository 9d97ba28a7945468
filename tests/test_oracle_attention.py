"""Pins for the oracle's float64 attention (CPU only).

Pinned against: brute-force Python loops (math.fsum, no max subtraction) on
tiny inputs, torch's float64 scaled_dot_product_attention (a library routine)
for unmasked / causal / explicitly masked cases, scipy's logsumexp for the
LSE, a two-key closed form, and the invariants a mistake anywhere would
break: rows of P sum to one, constant V returns V, a single visible key
returns its value row, a masked block contributes nothing, causal row 0 is
v_0, GQA equals duplicated KV heads, paged equals contiguous.
"""

import math

import numpy as np
import pytest

from oracle import attention as A


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _brute(q, k, v, scale, causal, block_mask, block):
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    o = np.zeros((B, Sq, Hq, v.shape[3]))
    lse = np.full((B, Hq, Sq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            for i in range(Sq):
                w = []
                for j in range(Skv):
                    ok = True
                    if causal and j > i + (Skv - Sq):
                        ok = False
                    if block_mask is not None and not block_mask[b, hk, i // block, j // block]:
                        ok = False
                    if ok:
                        s = scale * math.fsum(q[b, i, h, d] * k[b, j, hk, d] for d in range(D))
                        w.append((j, math.exp(s)))
                if not w:
                    continue
                den = math.fsum(e for _, e in w)
                for d in range(v.shape[3]):
                    o[b, i, h, d] = math.fsum(e * v[b, j, hk, d] for j, e in w) / den
                lse[b, h, i] = math.log(den)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Skv", [(5, 5), (7, 11), (11, 6), (16, 16)])
def test_brute_force_tiny(causal, Sq, Skv):
    rng = np.random.default_rng(10 + Sq + Skv)
    B, Hq, Hkv, D = 2, 4, 2, 8
    q, k, v = _rand(rng, B, Sq, Hq, D), _rand(rng, B, Skv, Hkv, D), _rand(rng, B, Skv, Hkv, D)
    block = 4
    bm = rng.random((B, Hkv, -(-Sq // block), -(-Skv // block))) < 0.6
    for mask in (None, bm):
        o, lse = A.attention(q, k, v, 0.37, causal, mask, block)
        ob, lseb = _brute(q, k, v, 0.37, causal, mask, block)
        assert np.allclose(o, ob, atol=1e-13, rtol=1e-12)
        fin = np.isfinite(lseb)
        assert np.array_equal(np.isfinite(lse), fin)
        assert np.allclose(lse[fin], lseb[fin], atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_qk_dim_differs_from_v_dim(causal):
    # The QK head dim and the V head dim are separate (192 / 128 in the wider
    # head-dim variant, 12 / 8 here): O takes V's width, scores sum over QK's.
    rng = np.random.default_rng(31)
    B, Sq, Skv, Hq, Hkv, Dqk, Dv = 1, 9, 13, 4, 2, 12, 8
    q, k, v = _rand(rng, B, Sq, Hq, Dqk), _rand(rng, B, Skv, Hkv, Dqk), _rand(rng, B, Skv, Hkv, Dv)
    o, lse = A.attention(q, k, v, 1 / math.sqrt(Dqk), causal)
    ob, lseb = _brute(q, k, v, 1 / math.sqrt(Dqk), causal, None, 4)
    assert o.shape == (B, Sq, Hq, Dv)
    assert np.allclose(o, ob, atol=1e-13, rtol=1e-12)
    fin = np.isfinite(lseb)
    assert np.allclose(lse[fin], lseb[fin], atol=1e-12)


def test_two_key_closed_form():
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    v = np.array([[2.0, -1.0], [4.0, 3.0]]).reshape(1, 2, 1, 2)
    o, lse = A.attention(q, k, v, 1.0)
    p0 = math.e / (math.e + 1.0)
    assert np.allclose(o[0, 0, 0], [2 * p0 + 4 * (1 - p0), -p0 + 3 * (1 - p0)], atol=1e-15)
    assert abs(lse[0, 0, 0] - math.log(math.e + 1.0)) < 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_float64(causal):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(11)
    B, S, H, D = 2, 300, 3, 64
    q, k, v = _rand(rng, B, S, H, D), _rand(rng, B, S, H, D), _rand(rng, B, S, H, D)
    o, _ = A.attention(q, k, v, 1 / 8, causal)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=1 / 8)
    assert np.allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


@pytest.mark.parametrize("Sq,Skv", [(200, 330), (1100, 1300)])
def test_matches_torch_sdpa_with_block_mask_and_bottom_right_causal(Sq, Skv):
    """1100 query rows span three of the oracle's 512-row chunks (a boundary bug
    in the chunking shows only there)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(12 + Sq)
    B, H, D, blk = 1, 2, 32, 64
    q, k, v = _rand(rng, B, Sq, H, D), _rand(rng, B, Skv, H, D), _rand(rng, B, Skv, H, D)
    bm = rng.random((B, H, -(-Sq // blk), -(-Skv // blk))) < 0.5
    bm[..., -1] = True  # keep every row alive
    o, _ = A.attention(q, k, v, 0.2, True, bm, blk)
    # explicit boolean mask built independently of the oracle's helper
    i = np.arange(Sq)[:, None]
    j = np.arange(Skv)[None, :]
    allowed = np.zeros((B, H, Sq, Skv), dtype=bool)
    for h in range(H):
        allowed[0, h] = (j <= i + (Skv - Sq)) & np.kron(bm[0, h], np.ones((blk, blk), bool))[:Sq, :Skv]
    alive = allowed.any(-1)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(allowed), scale=0.2)
    ref = ref.permute(0, 2, 1, 3).numpy()
    al = alive.transpose(0, 2, 1)
    assert np.allclose(o[al], ref[al], atol=1e-12)
    assert np.all(o[~al] == 0)


def test_lse_matches_scipy_logsumexp():
    from scipy.special import logsumexp

    rng = np.random.default_rng(13)
    q, k, v = _rand(rng, 1, 40, 1, 16), _rand(rng, 1, 70, 1, 16), _rand(rng, 1, 70, 1, 16)
    _, lse = A.attention(q, k, v, 0.5)
    ref = logsumexp(0.5 * q[0, :, 0] @ k[0, :, 0].T, axis=1)
    assert np.allclose(lse[0, 0], ref, atol=1e-12)


def test_rows_of_p_sum_to_one_and_masked_entries_are_zero():
    rng = np.random.default_rng(14)
    q, k = _rand(rng, 300, 32) * 3, _rand(rng, 400, 32) * 3
    bm = rng.random((3, 4)) < 0.5
    bm[:, 0] = True
    p = A.probabilities(q, k, 0.3, True, bm, 128)
    assert np.allclose(p.sum(1), 1.0, atol=1e-13)
    vis = A.visible_mask(300, 400, True, bm, 128)
    assert np.all(p[~vis] == 0)


def test_constant_v_returns_v():
    rng = np.random.default_rng(15)
    q, k = _rand(rng, 1, 257, 2, 64) * 4, _rand(rng, 1, 390, 2, 64) * 4
    row = rng.standard_normal(64)
    v = np.broadcast_to(row, (1, 390, 2, 64)).copy()
    o, _ = A.attention(q, k, v, 0.125, causal=True)
    assert np.allclose(o, row, atol=1e-12)


def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(16)
    Sq, Skv = 4, 9
    q, k, v = _rand(rng, 1, Sq, 1, 8), _rand(rng, 1, Skv, 1, 8), _rand(rng, 1, Skv, 1, 8)
    bm = np.zeros((1, 1, Sq, Skv), dtype=bool)  # block size 1: per-element mask
    for i in range(Sq):
        bm[0, 0, i, 2 * i] = True
    o, _ = A.attention(q, k, v, 1.0, False, bm, 1)
    for i in range(Sq):
        assert np.allclose(o[0, i, 0], v[0, 2 * i, 0], atol=1e-15)


def test_masked_block_contributes_nothing():
    rng = np.random.default_rng(17)
    S, blk = 512, 128
    q, k, v = _rand(rng, 1, S, 2, 32), _rand(rng, 1, S, 2, 32), _rand(rng, 1, S, 2, 32)
    bm = np.ones((1, 2, 4, 4), dtype=bool)
    bm[0, 1, :, 2] = False  # kv block 2 of kv head 1 dropped for every q block
    o1, l1 = A.attention(q, k, v, 0.2, False, bm, blk)
    k2, v2 = k.copy(), v.copy()
    k2[0, 256:384, 1] = rng.standard_normal((128, 32)) * 1e3
    v2[0, 256:384, 1] = rng.standard_normal((128, 32)) * 1e3
    o2, l2 = A.attention(q, k2, v2, 0.2, False, bm, blk)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_causal_row0_is_v0():
    rng = np.random.default_rng(18)
    q, k, v = _rand(rng, 2, 64, 3, 16), _rand(rng, 2, 64, 3, 16), _rand(rng, 2, 64, 3, 16)
    o, lse = A.attention(q, k, v, 0.25, causal=True)
    assert np.allclose(o[:, 0], v[:, 0], atol=1e-15)
    assert np.allclose(lse[:, :, 0], 0.25 * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]), atol=1e-14)


def test_gqa_equals_duplicated_kv_heads():
    rng = np.random.default_rng(19)
    B, S, Hq, Hkv, D = 1, 130, 8, 2, 16
    q, k, v = _rand(rng, B, S, Hq, D), _rand(rng, B, S, Hkv, D), _rand(rng, B, S, Hkv, D)
    o, lse = A.attention(q, k, v, 0.3, True)
    kd, vd = np.repeat(k, Hq // Hkv, axis=2), np.repeat(v, Hq // Hkv, axis=2)
    o2, lse2 = A.attention(q, kd, vd, 0.3, True)
    assert np.allclose(o, o2, atol=1e-14) and np.allclose(lse, lse2, atol=1e-14)
    # head h must use kv head h // 4: swapping the kv heads changes exactly the right heads
    o3, _ = A.attention(q, k[:, :, ::-1], v[:, :, ::-1], 0.3, True)
    assert not np.allclose(o3[:, :, :4], o[:, :, :4])


def test_paged_gather_equals_contiguous():
    rng = np.random.default_rng(20)
    B, Skv, H, D, page = 2, 200, 2, 8, 64
    npages = 4 * B
    pool = rng.standard_normal((npages, page, H, D))
    pt = rng.permutation(npages).reshape(B, 4)
    seq = A.gather_paged(pool, pt, Skv)
    for b in range(B):
        for t in range(Skv):
            assert np.array_equal(seq[b, t], pool[pt[b, t // page], t % page])


def test_fully_masked_rows_give_zero_and_minus_inf():
    rng = np.random.default_rng(21)
    q, k, v = _rand(rng, 1, 10, 1, 4), _rand(rng, 1, 4, 1, 4), _rand(rng, 1, 4, 1, 4)
    o, lse = A.attention(q, k, v, 1.0, causal=True)  # Sq > Skv: rows 0..5 see nothing
    assert np.all(o[0, :6] == 0) and np.all(np.isneginf(lse[0, 0, :6]))
    assert np.allclose(o[0, 6, 0], v[0, 0, 0])


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_equal_full_attention(causal):
    rng = np.random.default_rng(22)
    Sq, Skv, D, blk = 300, 420, 16, 64
    q, k, v = _rand(rng, 1, Sq, 1, D), _rand(rng, 1, Skv, 1, D), _rand(rng, 1, Skv, 1, D)
    bm = rng.random((1, 1, -(-Sq // blk), -(-Skv // blk))) < 0.6
    bm[..., -1] = True
    o, lse = A.attention(q, k, v, 0.3, causal, bm, blk)
    rows = np.array([0, 1, 63, 64, 150, 299])
    o2, lse2 = A.attention_rows(q[0, rows, 0], rows, k[0, :, 0], v[0, :, 0], 0.3, Sq, causal, bm[0, 0], blk)
    assert np.allclose(o2, o[0, rows, 0], atol=1e-14)
    fin = np.isfinite(lse[0, 0, rows])
    assert np.array_equal(np.isfinite(lse2), fin) and np.allclose(lse2[fin], lse[0, 0, rows][fin], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_probabilities_times_v_equals_brute_force(causal):
    """The invariant tests' helper: its P times V is the brute-force output."""
    rng = np.random.default_rng(23)
    Sq, Skv, D, blk = 9, 13, 6, 4
    q, k, v = _rand(rng, 1, Sq, 1, D), _rand(rng, 1, Skv, 1, D), _rand(rng, 1, Skv, 1, D)
    bm = rng.random((1, 1, -(-Sq // blk), -(-Skv // blk))) < 0.7
    bm[..., -1] = True
    p = A.probabilities(q[0, :, 0], k[0, :, 0], 0.7, causal, bm[0, 0], blk)
    o_ref, _ = _brute(q, k, v, 0.7, causal, bm, blk)
    assert np.allclose(p @ v[0, :, 0], o_ref[0, :, 0], atol=1e-13)
