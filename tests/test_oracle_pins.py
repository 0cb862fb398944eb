"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a hand-written golden mask, closed forms, a library routine on a
case where KSA reduces to it, or a second mechanism (the decode cache) that
the report says encodes the same visibility rule.

Citations: "Kwai Summary Attention Technical Report" (sections 2.2.1, 2.2.2,
2.3.1, Eqs. (1)-(3), (9), (10), Figures 3 and 4, Tables 1 and 3).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------------------
# Visibility
# ---------------------------------------------------------------------------
def test_fig3_toy_mask_matches_hand_written_golden():
    """Figure 3's toy (k=4, C=1, 16 text tokens): the predicate's dense mask
    equals the mask written out by hand from the rules of sections 2.2.1-2.2.2."""
    rows = []
    with open(os.path.join(GOLDEN, "fig3_toy_mask_k4_C1.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            bits = line.split()[0]
            rows.append([int(ch) for ch in bits])
    golden = np.array(rows, dtype=np.uint8)
    assert golden.shape == (20, 20)
    np.testing.assert_array_equal(oracle.dense_mask(16, 4, 1), golden)


def _closed_form_pairs(n, k, C):
    """Per-head visible pairs summed chunk by chunk: a text row at offset r of
    chunk c sees min(c, C)*k + r + 1 window keys and max(0, c - C) summaries;
    each complete chunk's summary sees k + 1 keys."""
    tot = 0
    nchunks = (n + k - 1) // k
    for c in range(nchunks):
        rows = min(k, n - c * k)
        tot += rows * min(c, C) * k + rows * (rows + 1) // 2 + rows * max(0, c - C)
    return tot + (n // k) * (k + 1)


@pytest.mark.parametrize("n,k,C,expect", [
    (256, 8, 2, 8824),            # the small prefill case (2 q / 1 kv heads, d 64)
    (32768, 8, 8, 69109792),      # the Qwen3-4B-shaped prefill case
])
def test_pair_counts_closed_form(n, k, C, expect):
    assert _closed_form_pairs(n, k, C) == expect
    assert lib_count(n, k, C) == expect


def lib_count(n, k, C):
    return int(oracle.lib().oracle_count_pairs(n, k, C))


def test_pair_counts_varlen_closed_form():
    lens = (131072, 65536, 16384, 4000)
    assert sum(lib_count(n, 8, 16) for n in lens) == 1385339220
    lens = (131072, 65536, 16384, 4003)
    assert sum(lib_count(n, 8, 16) for n in lens) == sum(_closed_form_pairs(n, 8, 16) for n in lens)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("C", [0, 1, 2, 100])
def test_mask_sum_equals_enumerated_keys(k, C):
    """Brute force over every (query, key) pair of the augmented sequence
    agrees with the key-set enumeration the attention uses, for all n <= 40."""
    for n in range(0, 41):
        mask = oracle.dense_mask(n, k, C)
        assert int(mask.sum()) == lib_count(n, k, C) == _closed_form_pairs(n, k, C)


def test_mask_structure_properties():
    """Properties the report states in words: a summary sees exactly its own
    chunk (k text) and itself; no text token sees an in-window summary; every
    past chunk is either fully visible as text or visible via its summary
    (section 2.2.2, 'clean partition' under Figure 4)."""
    for k, C in [(4, 1), (3, 2), (8, 0), (2, 5)]:
        n = 7 * k + (k // 2)
        m = n // k
        for i in range(n):
            c = i // k
            for cc in range(c):  # every fully past chunk
                text_vis = [oracle.visible(n, k, C, 0, i, 0, p) for p in range(cc * k, cc * k + k)]
                sum_vis = oracle.visible(n, k, C, 0, i, 1, cc)
                assert all(text_vis) != sum_vis or (all(text_vis) and not sum_vis)
                assert all(text_vis) or not any(text_vis)  # never a partial chunk
                assert all(text_vis) ^ sum_vis               # exactly one route
            # nothing of the future
            for p in range(i + 1, n):
                assert not oracle.visible(n, k, C, 0, i, 0, p)
            for j in range(c, m):
                assert not oracle.visible(n, k, C, 0, i, 1, j)
        for j in range(m):
            seen = [p for p in range(n) if oracle.visible(n, k, C, 1, j, 0, p)]
            assert seen == list(range(j * k, j * k + k))
            assert [jj for jj in range(m) if oracle.visible(n, k, C, 1, j, 1, jj)] == [j]


# ---------------------------------------------------------------------------
# Attention values
# ---------------------------------------------------------------------------
def _sdpa(q, k, v, causal, scale):
    """torch fp64 SDPA on [H, L, d] (GQA already expanded)."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        is_causal=causal, scale=scale)[0].numpy()


@pytest.mark.parametrize("n,k,Hq,Hkv,d", [(37, 4, 4, 2, 16), (64, 8, 2, 1, 32), (21, 1, 3, 3, 8)])
def test_text_rows_reduce_to_causal_attention(n, k, Hq, Hkv, d):
    """With C >= n/k no chunk ever leaves the window, so Eq. (3) has no
    summaries and the text rows are causal full attention over the text
    (the teacher of Eq. (9) with a causal mask)."""
    rng = np.random.default_rng(1)
    m = n // k
    qt, kt, vt = _rand(rng, n, Hq, d), _rand(rng, n, Hkv, d), _rand(rng, n, Hkv, d)
    qs, ks, vs = _rand(rng, m, Hq, d), _rand(rng, m, Hkv, d), _rand(rng, m, Hkv, d)
    scale = 1 / math.sqrt(d)
    ot, lt, _, _ = oracle.ksa_attention(n, k, n // k + 1, qt, kt, vt, qs, ks, vs)
    G = Hq // Hkv
    ref = _sdpa(qt.transpose(1, 0, 2), np.repeat(kt, G, 1).transpose(1, 0, 2),
                np.repeat(vt, G, 1).transpose(1, 0, 2), True, scale).transpose(1, 0, 2)
    np.testing.assert_allclose(ot, ref, rtol=0, atol=1e-12)
    # LSE: log-sum-exp of the causal scores
    s = np.einsum("ihd,jhd->hij", qt, np.repeat(kt, G, 1)) * scale
    s = np.where(np.tril(np.ones((n, n), bool))[None], s, -np.inf)
    np.testing.assert_allclose(lt, torch.logsumexp(torch.from_numpy(s), -1).numpy().T, atol=1e-12)


def test_summary_rows_are_softmax_over_own_chunk():
    """s_j attends to t_{jk}..t_{jk+k-1} and s_j (k+1 keys): plain SDPA on
    that slice (section 2.2.1 summary rule, with the self key of Figure 4c)."""
    rng = np.random.default_rng(2)
    n, k, C, Hq, Hkv, d = 43, 5, 1, 4, 2, 16
    m = n // k
    qt, kt, vt = _rand(rng, n, Hq, d), _rand(rng, n, Hkv, d), _rand(rng, n, Hkv, d)
    qs, ks, vs = _rand(rng, m, Hq, d), _rand(rng, m, Hkv, d), _rand(rng, m, Hkv, d)
    _, _, os_, ls = oracle.ksa_attention(n, k, C, qt, kt, vt, qs, ks, vs)
    G = Hq // Hkv
    for j in range(m):
        keys = np.concatenate([kt[j * k:(j + 1) * k], ks[j:j + 1]], 0)
        vals = np.concatenate([vt[j * k:(j + 1) * k], vs[j:j + 1]], 0)
        keys, vals = np.repeat(keys, G, 1), np.repeat(vals, G, 1)
        ref = _sdpa(qs[j][:, None], keys.transpose(1, 0, 2), vals.transpose(1, 0, 2), False,
                    1 / math.sqrt(d))[:, 0]
        np.testing.assert_allclose(os_[j], ref, atol=1e-12)


@pytest.mark.parametrize("k,C", [(4, 1), (3, 2), (1, 0), (8, 0), (2, 3)])
def test_one_hot_values_reveal_the_visible_set(k, C):
    """With q = 0 the softmax is uniform over the visible keys, and with a
    one-hot value per key the output is 1/count exactly on the keys the
    dense predicate marks.  Pins the enumeration in the attention against
    the brute-force mask, both directions."""
    n = 6 * k + (k - 1 if k > 1 else 0)
    m = n // k
    L = n + m
    mask = oracle.dense_mask(n, k, C)
    d = L
    # one-hot V: key with augmented index a carries e_a
    text_aug = np.array([i + i // k for i in range(n)])
    sum_aug = np.array([j * (k + 1) + k for j in range(m)])
    vt = np.zeros((n, 1, d)); vt[np.arange(n), 0, text_aug] = 1
    vs = np.zeros((m, 1, d)); vs[np.arange(m), 0, sum_aug] = 1
    z_t, z_s = np.zeros((n, 1, d)), np.zeros((m, 1, d))
    ot, lt, os_, ls = oracle.ksa_attention(n, k, C, z_t, z_t, vt, z_s, z_s, vs)
    for i in range(n):
        row = mask[text_aug[i]]
        np.testing.assert_allclose(ot[i, 0], row / row.sum(), atol=1e-15)
        assert abs(lt[i, 0] - math.log(row.sum())) < 1e-12
    for j in range(m):
        row = mask[sum_aug[j]]
        np.testing.assert_allclose(os_[j, 0], row / row.sum(), atol=1e-15)
        assert abs(ls[j, 0] - math.log(k + 1)) < 1e-12


def test_single_visible_key_returns_its_value():
    """t_0 sees only itself: its output is v_0 whatever q and k are."""
    rng = np.random.default_rng(3)
    n, k, C, d = 9, 4, 1, 8
    qt, kt, vt = _rand(rng, n, 1, d), _rand(rng, n, 1, d), _rand(rng, n, 1, d)
    m = n // k
    qs, ks, vs = _rand(rng, m, 1, d), _rand(rng, m, 1, d), _rand(rng, m, 1, d)
    ot, lt, _, _ = oracle.ksa_attention(n, k, C, qt, kt, vt, qs, ks, vs)
    np.testing.assert_allclose(ot[0, 0], vt[0, 0], atol=1e-15)
    assert abs(lt[0, 0] - qt[0, 0] @ kt[0, 0] / math.sqrt(d)) < 1e-12


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------
def test_rope_identity_at_position_zero_and_norm_preserving():
    rng = np.random.default_rng(4)
    x = _rand(rng, 5, 3, 16)
    out0 = oracle.rope(x, np.zeros(5, np.int64), 1e6)
    np.testing.assert_array_equal(out0, x)
    out = oracle.rope(x, np.array([1, 7, 100, 4095, 1 << 20]), 1e6)
    h = 8
    np.testing.assert_allclose(out[..., :h] ** 2 + out[..., h:] ** 2,
                               x[..., :h] ** 2 + x[..., h:] ** 2, rtol=1e-13)


def test_rope_frequency_schedule_closed_form():
    """theta = 1e6 (Table 3), d = 128: pair r turns by pos * theta^(-2r/d).
    Pair 0 turns by pos radians; pair d/4 = 32 turns by pos * 1e-3 radians,
    so position 1000 turns it by exactly 1 radian; rotate-half pairs element
    r with element r + d/2."""
    d = 128
    x = np.zeros((1, 1, d))
    x[0, 0, 0] = 1.0
    x[0, 0, 32] = 1.0
    out = oracle.rope(x, np.array([1000]), 1e6)[0, 0]
    assert abs(out[0] - math.cos(1000.0)) < 1e-12 and abs(out[64] - math.sin(1000.0)) < 1e-12
    assert abs(out[32] - math.cos(1.0)) < 1e-12 and abs(out[96] - math.sin(1.0)) < 1e-12
    assert np.count_nonzero(np.abs(out) > 1e-15) == 4


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(5)
    d = 32
    q, k = _rand(rng, 1, 1, d), _rand(rng, 1, 1, d)
    def score(pq, pk):
        return float(oracle.rope(q, np.array([pq]), 1e6)[0, 0] @ oracle.rope(k, np.array([pk]), 1e6)[0, 0])
    assert abs(score(10, 3) - score(1010, 1003)) < 1e-10
    assert abs(score(70000, 5) - score(69995, 0)) < 1e-9


def test_summary_position_is_last_text_position_of_its_chunk():
    assert list(oracle.summary_positions(19, 4)) == [3, 7, 11, 15]
    assert list(oracle.summary_positions(8, 8)) == [7]


# ---------------------------------------------------------------------------
# Decode cache model (section 2.3.1, Figure 4)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("k,C", [(4, 2), (3, 1), (8, 0), (2, 4), (1, 3)])
def test_cache_decode_equals_prefill_rows(k, C):
    """Decode step t over the single contiguous slice equals row t of the
    masked prefill (Eq. (3) enumeration) -- two different mechanisms that the
    report says encode the same rule ('the cache layout itself inherently
    encodes the visibility rule').  Covers ring wrap-around (m > C) and the
    summary steps."""
    rng = np.random.default_rng(10 + k * 7 + C)
    Hq, Hkv, d = 4, 2, 8
    n = 11 * k + (k // 2)
    m = n // k
    qt, kt, vt = _rand(rng, n, Hq, d), _rand(rng, n, Hkv, d), _rand(rng, n, Hkv, d)
    qs, ks, vs = _rand(rng, m, Hq, d), _rand(rng, m, Hkv, d), _rand(rng, m, Hkv, d)
    ot, lt, os_, ls = oracle.ksa_attention(n, k, C, qt, kt, vt, qs, ks, vs)
    cache = oracle.Cache(k, C, Hkv, d, cap=m)
    for i in range(n):
        assert cache.append_text(kt[i], vt[i]) == 0
        lo, hi = cache.slice(oracle.TEXT)
        assert 0 <= lo < hi <= cache.S
        o, l = cache.decode(oracle.TEXT, qt[i])
        np.testing.assert_allclose(o, ot[i], atol=1e-12)
        np.testing.assert_allclose(l, lt[i], atol=1e-12)
        if (i + 1) % k == 0:
            j = (i + 1) // k - 1
            assert cache.append_text(kt[i], vt[i]) == -1      # chunk full: summary first
            assert cache.append_summary(ks[j], vs[j]) == 0
            o, l = cache.decode(oracle.SUMMARY, qs[j])
            np.testing.assert_allclose(o, os_[j], atol=1e-12)
            np.testing.assert_allclose(l, ls[j], atol=1e-12)
    assert cache.n_text == n and cache.m == m


@pytest.mark.parametrize("k,C,n0,pending,T", [
    (4, 2, 0, False, 23),    # a block from an empty cache
    (4, 2, 10, False, 13),   # open chunk with 2 cached tokens, ring wraps inside the block
    (4, 2, 12, True, 9),     # chunk 2 complete, its summary still to come
    (3, 1, 7, False, 0),     # an empty block
    (8, 0, 16, True, 0),     # only the pending summary
    (1, 2, 5, False, 6),     # k = 1: every token completes a chunk
    (2, 4, 9, False, 21),    # w larger than the chunks before the block
])
def test_chunk_rows_equal_decode_steps(k, C, n0, pending, T):
    """A chunked prefill's rows (by definition, prefill rows n0 .. n0+T-1 and
    the summaries of the chunks the block completes) equal the decode steps
    of the same tokens against the cache of the first n0 -- two mechanisms
    (Eq. (3) enumeration vs the slot map of Figure 4) that must agree."""
    rng = np.random.default_rng(100 + 13 * k + n0 + T)
    Hq, Hkv, d, theta = 4, 2, 8, 1e6
    n1 = n0 + T
    m1 = n1 // k
    m0 = n0 // k - (1 if pending else 0)
    qt, kt, vt = _rand(rng, n1, Hq, d), _rand(rng, n1, Hkv, d), _rand(rng, n1, Hkv, d)
    qs, ks, vs = _rand(rng, m1, Hq, d), _rand(rng, m1, Hkv, d), _rand(rng, m1, Hkv, d)
    ref = oracle.ksa_prefill_chunk(n0, m0, T, k, C, qt, kt, vt, qs, ks, vs, theta)
    assert ref.text_o.shape[0] == T and ref.sum_o.shape[0] == m1 - m0
    pt, ps = oracle.text_positions(n1), oracle.summary_positions(n1, k)
    rq, rk = oracle.rope(qt, pt, theta), oracle.rope(kt, pt, theta)
    sq = oracle.rope(qs, ps, theta) if m1 else qs
    sk = oracle.rope(ks, ps, theta) if m1 else ks
    cache = oracle.Cache(k, C, Hkv, d, cap=m1 + 1)
    for i in range(n0):
        assert cache.append_text(rk[i], vt[i]) == 0
        if (i + 1) % k == 0 and (i + 1) // k - 1 < m0:
            assert cache.append_summary(sk[(i + 1) // k - 1], vs[(i + 1) // k - 1]) == 0
    assert cache.n_text == n0 and cache.m == m0
    if pending:
        assert cache.append_summary(sk[m0], vs[m0]) == 0
        o, l = cache.decode(oracle.SUMMARY, sq[m0])
        np.testing.assert_allclose(o, ref.sum_o[0], atol=1e-12)
        np.testing.assert_allclose(l, ref.sum_lse[0], atol=1e-12)
    for t in range(T):
        i = n0 + t
        assert cache.append_text(rk[i], vt[i]) == 0
        o, l = cache.decode(oracle.TEXT, rq[i])
        np.testing.assert_allclose(o, ref.text_o[t], atol=1e-12)
        np.testing.assert_allclose(l, ref.text_lse[t], atol=1e-12)
        if (i + 1) % k == 0:
            j = (i + 1) // k - 1
            assert cache.append_summary(sk[j], vs[j]) == 0
            o, l = cache.decode(oracle.SUMMARY, sq[j])
            np.testing.assert_allclose(o, ref.sum_o[j - m0], atol=1e-12)
            np.testing.assert_allclose(l, ref.sum_lse[j - m0], atol=1e-12)
    assert cache.n_text == n1 and cache.m == m1


def test_cache_slot_map_contents():
    """The documented slot map, checked slot by slot after a run that wraps
    the ring: scratch = newest summary, summaries in order from slot
    1+k+C*k, ring block c % C holds chunk c (block copy, reversed order),
    current chunk right-aligned against the ring."""
    k, C, Hkv, d = 3, 2, 1, 2
    n = 5 * k + 2
    m = n // k
    tok = np.arange(n, dtype=np.float64)
    cache = oracle.Cache(k, C, Hkv, d, cap=m + 1)
    for i in range(n):
        cache.append_text(np.full((Hkv, d), tok[i]), np.full((Hkv, d), -tok[i]))
        if (i + 1) % k == 0:
            j = (i + 1) // k - 1
            cache.append_summary(np.full((Hkv, d), 1000.0 + j), np.full((Hkv, d), -1000.0 - j))
    K = cache.K()[:, 0, 0]
    assert K[0] == 1000 + (m - 1)
    for j in range(m):
        assert K[1 + k + C * k + j] == 1000 + j
    for c in range(m - C, m):
        b = c % C
        for r in range(k):
            assert K[1 + k + b * k + (k - 1 - r)] == c * k + r
    f = n - m * k
    for r in range(f):
        assert K[k - r] == m * k + r
    lo, hi = cache.slice(oracle.TEXT)
    assert (lo, hi) == (k - f + 1, 1 + k + C * k + (m - C))


def test_cache_capacity_and_order_errors():
    cache = oracle.Cache(2, 1, 1, 2, cap=1)
    row = np.ones((1, 2))
    assert cache.append_summary(row, row) == -1  # chunk not complete
    cache.append_text(row, row); cache.append_text(row, row)
    assert cache.append_summary(row, row) == 0
    cache.append_text(row, row); cache.append_text(row, row)
    assert cache.append_summary(row, row) == -3  # buffer full


def test_table1_cache_ratios():
    """Table 1: with k = 8 the KSA cache grows at 1/k of full attention; with
    GQA (g = 8 of h = 128 heads) that is 1/k * g/h = 0.78125% of MHA.  The
    cache's slot count per sequence is 1 + k + C*k + n/k, so the ratio tends
    to 1/k as n grows."""
    k, C = 8, 8
    n = 1 << 24
    slots = oracle.cache_slots(k, C, n // k)
    assert abs(slots / n - 1 / k) < 1e-4
    h, g = 128, 8
    assert abs(slots * g / (n * h) - 0.0078125) < 1e-6


# ---------------------------------------------------------------------------
# KSA over an MLA latent cache (section 3.2, Eq. (6); MLA of section 3.1)
# ---------------------------------------------------------------------------
def test_mla_absorbed_equals_explicit_per_head_attention():
    """The oracle's latent decode (absorbed MLA as multi-query attention over
    [c, r] rows) equals MLA computed the explicit way: per-head keys
    [W_UK c, r] and values W_UV c rebuilt from random up-projections, softmax
    over the visible slots, then compared after mapping the latent output
    through W_UV."""
    rng = np.random.default_rng(77)
    k, C, H, d_c, d_r, d_nope, d_v, theta = 4, 2, 3, 16, 8, 6, 5, 1e6
    n = 6 * k + 3
    m = n // k
    cap = m + 1
    lat_t = rng.standard_normal((n, d_c + d_r))
    lat_s = rng.standard_normal((m, d_c + d_r))
    W_uk = rng.standard_normal((H, d_nope, d_c))
    W_uv = rng.standard_normal((H, d_v, d_c))
    q_nope = rng.standard_normal((H, d_nope))
    q_rope = rng.standard_normal((H, d_r))
    scale = 1.0 / math.sqrt(d_nope + d_r)
    cache = oracle.Cache(k, C, 1, d_c + d_r, cap)
    Kt, Vt = oracle.mla_kv_rows(lat_t, np.arange(n), theta, d_c)
    Ks, Vs = oracle.mla_kv_rows(lat_s, oracle.summary_positions(n, k), theta, d_c)
    for i in range(n):
        cache.append_text(Kt[i:i + 1], Vt[i:i + 1])
        if (i + 1) % k == 0:
            cache.append_summary(Ks[(i + 1) // k - 1:(i + 1) // k], Vs[(i + 1) // k - 1:(i + 1) // k])
    # absorbed: q_c = W_UK^T q_nope
    q_abs = np.concatenate([np.einsum("hnc,hn->hc", W_uk, q_nope), q_rope], axis=1)
    o_lat, lse = oracle.mla_decode_image(k, C, cap, n, m, oracle.TEXT, cache.K()[:, 0], q_abs, scale, theta, d_c)
    # explicit: visible keys of text token n-1 by the rule (Eqs. (2)-(3))
    i = n - 1
    c = i // k
    txt = [j for j in range(max(0, c - C) * k, i + 1)]
    sm = [j for j in range(max(0, c - C))]
    rows = [Kt[j] for j in txt] + [Ks[j] for j in sm]
    qr = oracle.rope(q_rope[None], np.array([i]), theta)[0]
    for h in range(H):
        keys = np.stack([np.concatenate([W_uk[h] @ r[:d_c], r[d_c:]]) for r in rows])
        vals = np.stack([W_uv[h] @ r[:d_c] for r in rows])
        s = scale * keys @ np.concatenate([q_nope[h], qr[h]])
        p = np.exp(s - s.max())
        want = (p / p.sum()) @ vals
        np.testing.assert_allclose(W_uv[h] @ o_lat[h], want, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[h], s.max() + np.log(np.exp(s - s.max()).sum()), atol=1e-12)


def test_mla_table1_cache_ratio():
    """Eq. (6) against Table 1's setting (h = 128, d = 128, d_c = 512,
    d_r = 64, k = 8): KSA + MLA keeps (d_c + d_r) / k values per token, 576/8
    = 72, i.e. 72 / (2 h d) = 0.22 % of MHA's 2 h d per token."""
    h, d, d_c, d_r, k = 128, 128, 512, 64, 8
    per_token = (d_c + d_r) / k
    assert per_token == 72
    assert round(100 * per_token / (2 * h * d), 2) == 0.22
