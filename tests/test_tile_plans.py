"""CPU checks of the CUDA library's work decomposition against the KSA mask.

The block-sparse kernels never look at the L x L mask: each one derives its
list of tiles from chunk coordinates.  The parity tests on the GPU show that
the outputs are right; a tile list that reads a tile too many still passes
them.  These tests run the kernels' own index functions, compiled for the
host (tests/plan_harness.cu), over many shapes, and check each list against
the oracle's dense mask:
  - every row (sequence, q head, text token) belongs to exactly one work item;
  - every key that a row of a work item sees lies in one of its tiles;
  - every tile holds at least one key that some row of the item sees, so no
    fully masked tile is ever loaded or multiplied ("Kwai Summary Attention
    Technical Report", section 2.3 "Kernel Design": only block pairs the mask
    does not zero out entirely are computed);
  - the backward's key tiles split the keys, and the text query range of
    each tile is exactly the span of the queries that see it; its query
    tiles split the text rows and hold what those rows see; its grids and
    workspace bound the work lists;
  - the chunked prefill's gathered buffers hold what its work items read,
    within the sizes the workspace reserves, and every key its rows see is
    read from the cache slot where the oracle's cache holds that key (or
    from the block's own input rows);
  - the decode's live slots match the oracle's cache (section 2.3.1,
    Figure 4) in every reachable state, and unreachable states are refused.
The visibility rule is section 2.2.1 (summaries) and section 2.2.2,
Eqs. (2)-(3) (text).
"""
from __future__ import annotations

import functools
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "plan_harness.cu")
BM = BN = BK = 128   # query-tile rows, K/V-tile keys (forward), key-tile keys (backward)
TEXT, SUMMARY = 0, 1


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    exe = str(tmp_path_factory.mktemp("plan") / "plan_harness")
    # PTX only: the kernels are compiled along with the host code, never run
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=compute_100a", "-std=c++17", "-O1",
                           "-o", exe, SRC])
    proc = subprocess.Popen([exe], stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True)

    def query(*words):
        proc.stdin.write(" ".join(str(x) for x in words) + "\n")
        proc.stdin.flush()
        rows = []
        while True:
            line = proc.stdout.readline()
            assert line, "harness exited"
            line = line.strip()
            if line == "end":
                return rows
            assert line not in ("bad query", "unsupported"), (words, line)
            rows.append([int(x) for x in line.split()])

    yield query
    proc.stdin.close()
    proc.wait(timeout=30)


# ---------------------------------------------------------------------------
# The mask, as [text query, text key] and [text query, summary] booleans
# ---------------------------------------------------------------------------
@functools.lru_cache(maxsize=None)
def text_views(n: int, k: int, w: int):
    m = n // k
    M = oracle.dense_mask(n, k, w).astype(bool)
    t = np.arange(n)
    pt = (t // k) * (k + 1) + t % k          # Eq. (1) position of text token t
    ps = np.arange(m) * (k + 1) + k          # and of summary s_j
    return M[np.ix_(pt, pt)], M[np.ix_(pt, ps)]


def offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


# ---------------------------------------------------------------------------
# Forward work items
# ---------------------------------------------------------------------------
FIELDS = ("hkv", "h0", "b", "nb", "mb", "ncb", "qbase", "kvbase", "sbase", "c0", "cend", "cw_lo", "n_win", "T")


def check_items(rows, k, w, Hq, Hkv, seq, row_lo=None):
    """Checks the work items printed by the harness.  seq[b] = (ntot, first
    query chunk, first window chunk held or None, q-buffer / window-buffer
    chunk bases or None); row_lo[b]: the first row the call must produce."""
    W, Gp, HP, Tc, Tk = rows[0]
    items = [dict(zip(FIELDS, r)) for r in rows[1:]]
    G = Hq // Hkv
    assert len(items) == W
    assert Gp * HP == G and Gp * k * Tc <= BM and Tk == BN // k
    assert Gp == min(G, BM // k) and Tc == BM // (Gp * k)
    covered = {}
    for it in items:
        b = it["b"]
        ntot, cbeg, kvb, bases = seq[b]
        n, m, ncb = ntot, ntot // k, -(-ntot // k)
        assert (it["nb"], it["mb"], it["ncb"]) == (n, m, ncb)
        if bases is not None:
            assert (it["qbase"], it["kvbase"]) == bases
        assert it["hkv"] * G <= it["h0"] and it["h0"] + Gp <= (it["hkv"] + 1) * G
        assert (it["h0"] - it["hkv"] * G) % Gp == 0
        c0, cend = it["c0"], it["cend"]
        assert cbeg <= c0 < cend <= ncb and cend - c0 <= Tc
        assert (c0 - cbeg) % Tc == 0 and (cend == c0 + Tc or cend == ncb)
        for h in range(it["h0"], it["h0"] + Gp):
            for c in range(c0, cend):
                key = (b, h, c)
                assert key not in covered, ("row covered twice", key)
                covered[key] = True
        # keys the item's rows see, against its tiles
        vt, vs = text_views(n, k, w)
        r0, r1 = c0 * k, min(cend * k, n)
        seen_t = np.flatnonzero(vt[r0:r1].any(axis=0))
        seen_s = np.flatnonzero(vs[r0:r1].any(axis=0))
        cw_lo, n_win, T = it["cw_lo"], it["n_win"], it["T"]
        assert cw_lo == max(0, c0 - w)
        if kvb is not None:
            assert cw_lo >= kvb, "a window tile starts before the chunks the buffer holds"
            assert seen_t.size == 0 or (seen_t[0] >= kvb * k and seen_t[-1] < ncb * k)
        lo, hi = cw_lo * k, (cw_lo + n_win * Tk) * k
        assert seen_t.size and seen_t[0] >= lo and seen_t[-1] < hi, "a visible text key outside the window tiles"
        for j in range(n_win):
            a, z = lo + j * Tk * k, lo + (j + 1) * Tk * k
            assert np.any((seen_t >= a) & (seen_t < z)), ("fully masked window tile", it, j)
        n_sum = T - n_win
        assert n_sum >= 0
        assert seen_s.size == 0 or seen_s[-1] < n_sum * BN, "a visible summary outside the summary tiles"
        if seen_s.size:
            assert seen_s[0] == 0 and seen_s.size == seen_s[-1] + 1   # a prefix s_0 .. s_{ns-1}
        for j in range(n_sum):
            assert np.any((seen_s >= j * BN) & (seen_s < (j + 1) * BN)), ("fully masked summary tile", it, j)
    # every (sequence, q head, chunk) the call must produce
    for b, (ntot, cbeg, _, _) in enumerate(seq):
        ncb = -(-ntot // k)
        first = cbeg if row_lo is None else row_lo[b] // k
        for h in range(Hq):
            for c in range(first, ncb):
                assert (b, h, c) in covered, ("row not covered", b, h, c)
    return items


def fwd_case(harness, k, w, Hq, Hkv, seqlens):
    rows = harness("fwd", k, w, Hq, Hkv, len(seqlens), *seqlens)
    coff = offsets([-(-n // k) for n in seqlens])
    seq = [(n, 0, None, (int(coff[b]), int(coff[b]))) for b, n in enumerate(seqlens)]
    items = check_items(rows, k, w, Hq, Hkv, seq)
    for it in items:
        assert it["sbase"] == it["qbase"]
    return items


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 8, 12, 16, 24, 32, 64, 100, 128])
@pytest.mark.parametrize("w", [0, 1, 2, 5, 16])
def test_forward_items_cover_the_mask_and_skip_masked_tiles(harness, k, w):
    rng = np.random.default_rng(1000 * k + w)
    Hq, Hkv = [(8, 8), (16, 8), (32, 8), (64, 4)][(k + w) % 4]
    lens = [int(x) for x in rng.integers(1, 700 if k > 2 else 300, size=3)] + [k, k + 1, max(k - 1, 1)]
    fwd_case(harness, k, w, Hq, Hkv, lens)


@pytest.mark.parametrize("k,Hq,Hkv", [(8, 32, 8), (16, 128, 8), (64, 16, 1), (128, 8, 4), (7, 72, 4)])
def test_forward_items_split_heads_when_a_kv_group_exceeds_the_tile(harness, k, Hq, Hkv):
    """G k > 128: the q heads of a kv head split over several items, each
    with the same K/V tiles (Gp = 128 / k heads per item)."""
    items = fwd_case(harness, k, 3, Hq, Hkv, [900, 130, 1])
    G = Hq // Hkv
    if G * k > BM:
        assert max(it["h0"] - it["hkv"] * G for it in items) > 0


def test_forward_items_empty_sequences_and_heavy_first_order(harness):
    k, w = 8, 2
    lens = [0, 300, 0, 5, 0, 1200]
    items = fwd_case(harness, k, w, 32, 8, lens)
    assert all(it["b"] not in (0, 2, 4) for it in items)
    # round robin hands out the latest units of the last sequence first
    assert items[0]["b"] == 5 and items[0]["cend"] == -(-1200 // k)


# ---------------------------------------------------------------------------
# Chunked prefill: a block of T new tokens against a cache holding n0 / m0
# ---------------------------------------------------------------------------
def chunk_case(harness, k, w, Hq, Hkv, states):
    trip = [x for s in states for x in s]
    rows = harness("chunk", k, w, Hq, Hkv, len(states), *trip)
    B = len(states)
    per, tail, item_rows = rows[:B], rows[B], rows[B + 1:]
    sum_q, sum_kv, units, Lq, Lkv, Lunits, slot0 = tail
    assert slot0 == 1 + k + w * k
    # the gathered buffers and the unit list fit the workspace the call reserves
    assert sum_q <= Lq and sum_kv <= Lkv and units <= Lunits
    seq, row_lo = [], []
    for (n0, m0, T), (code, cb, kvb, ncb, qoff, kvoff) in zip(states, per):
        f0 = n0 - m0 * k
        valid = 0 <= f0 <= k and n0 >= 0 and m0 >= 0
        assert (code == 0) == valid, (n0, m0, T, code)
        if valid and T > 0:
            assert cb == n0 // k and ncb == -(-(n0 + T) // k)
            assert kvb == max(0, min(cb - w, m0))
            # the chunk of the first new summary is among the window chunks
            assert kvb <= m0
        seq.append((n0 + T, cb, kvb, (qoff - cb, kvoff - kvb)))
        row_lo.append(n0)
    active = [b for b, (s, p) in enumerate(zip(states, per)) if p[0] == 0 and s[2] > 0]
    check_items(item_rows, k, w, Hq, Hkv, [seq[b] if b in active else (0, 0, 0, None) for b in range(B)],
                row_lo=[row_lo[b] if b in active else 0 for b in range(B)])


@pytest.mark.parametrize("k,w", [(1, 0), (2, 3), (4, 1), (8, 2), (8, 8), (16, 4), (32, 1), (64, 2), (128, 0), (6, 3)])
def test_chunk_items_read_only_their_own_buffers(harness, k, w):
    rng = np.random.default_rng(77 + k * 10 + w)
    states = []
    for _ in range(5):
        n0 = int(rng.integers(0, 600))
        T = int(rng.integers(1, 400))
        states.append((n0, n0 // k, T))
    # a full chunk whose summary is still pending (f0 = k), a block that
    # starts on a chunk boundary, a one-token block, an empty block
    states += [(3 * k, 2, 5), (4 * k, 4, 2 * k), (k + 1, 1, 1), (50, 50 // k, 0)]
    chunk_case(harness, k, w, 32, 8, states)


def test_chunk_invalid_states_get_no_work(harness):
    k, w = 8, 2
    states = [(20, 1, 10),   # f0 = 12 > k
              (20, 3, 10),   # f0 < 0
              (16, 2, 30),   # valid: f0 = 0
              (-1, 0, 5)]
    chunk_case(harness, k, w, 32, 8, states)


# ---------------------------------------------------------------------------
# Backward key tiles
# ---------------------------------------------------------------------------
KT = ("b", "sum", "j0", "kcnt", "n", "m", "c0", "qlo", "qhi", "nq", "lead", "nsh")
QT = ("b", "n", "m", "c0", "q0", "qn", "c_first", "ns", "n_sum", "t_lo", "n_win")


def bwd_case(harness, k, w, Hq, Hkv, seqlens):
    rows = harness("bwd", k, w, Hq, Hkv, len(seqlens), *seqlens)
    ns, nt, nqs, split, max_tiles, dkv_grid, dq_grid, dkv_ctas = rows[0]
    G = Hq // Hkv
    # steps of 64 query positions when k divides 64, else of 128
    assert nqs == (64 if 64 % k == 0 else 128) and nqs % k == 0
    # launch bounds: the plan never needs more tiles, or CTAs, than reserved
    assert ns + nt <= max_tiles and dkv_ctas <= dkv_grid and nt <= dq_grid
    tiles = [dict(zip(KT, r)) for r in rows[1:1 + ns + nt]]
    shares = [list(zip(r[len(KT)::2], r[len(KT) + 1::2])) for r in rows[1:1 + ns + nt]]
    check_dq_tiles(rows[1 + ns + nt:], k, w, seqlens, nt)
    check_shares(tiles, shares, G, nqs, split)
    coff = offsets([-(-n // k) for n in seqlens])
    got_s = {b: [] for b in range(len(seqlens))}
    got_t = {b: [] for b in range(len(seqlens))}
    for i, T in enumerate(tiles):
        b = T["b"]
        n = seqlens[b]
        m = n // k
        assert (T["n"], T["m"], T["c0"]) == (n, m, coff[b])
        assert bool(T["sum"]) == (i < ns), "summary tiles come first"
        j0, kc = T["j0"], T["kcnt"]
        assert j0 % BK == 0 and 1 <= kc <= BK
        vt, vs = text_views(n, k, w)
        if T["sum"]:
            assert j0 + kc <= m and (kc == BK or j0 + kc == m)
            got_s[b].append(j0)
            q = np.flatnonzero(vs[:, j0:j0 + kc].any(axis=1))
        else:
            assert j0 + kc <= n and (kc == BK or j0 + kc == n)
            got_t[b].append(j0)
            q = np.flatnonzero(vt[:, j0:j0 + kc].any(axis=1))
        qlo, qhi = T["qlo"], T["qhi"]
        if q.size:
            assert (qlo, qhi) == (q[0], q[-1] + 1), ("query range not the span of the queries that see it", T)
        else:
            assert qhi <= qlo
        assert T["nq"] == (-(-(qhi - qlo) // nqs) if qhi > qlo else 0)
    for b, n in enumerate(seqlens):
        assert got_s[b] == list(range(0, n // k, BK))
        assert got_t[b] == list(range(0, n, BK))
    assert dkv_ctas == sum(T["nsh"] for T in tiles)


def check_shares(tiles, shares, G, nqs, split):
    """dk/dv shares: each tile's shares cut its nq query blocks into
    consecutive non-empty runs of at most split // G blocks (a CTA's steps
    are blocks x G heads, at most split); text tiles' shares start at the
    tile's first block; the summary tiles of one sequence cut the queries
    at common positions (a window grid of split // G blocks), so that the
    shares of different tiles over one window read the same Q and dO."""
    bpw = max(1, split // G)
    grid = {}
    for T, sh in zip(tiles, shares):
        assert len(sh) == T["nsh"]
        if T["nq"] == 0:
            assert sh == []
            continue
        assert sh[0][0] == 0 and sh[-1][1] == T["nq"]
        for (a0, a1), (b0, _) in zip(sh, sh[1:]):
            assert a1 == b0
        assert all(1 <= r1 - r0 <= bpw for r0, r1 in sh)
        if not T["sum"]:
            assert T["lead"] == 0 and len(sh) == -(-T["nq"] // bpw)
            continue
        assert 0 <= T["lead"] < bpw
        # the share starts after the first, and the start of the first
        # share's window (lead blocks before qlo), all on one grid
        cuts = {(T["qlo"] + r0 * nqs) % (bpw * nqs) for r0, _ in sh[1:]}
        cuts.add((T["qlo"] - T["lead"] * nqs) % (bpw * nqs))
        grid.setdefault(T["b"], set()).update(cuts)
    for b, cuts in grid.items():
        assert len(cuts) == 1, ("summary tiles of a sequence cut their queries on different grids", b, cuts)


def check_dq_tiles(rows, k, w, seqlens, nt):
    """dq: one CTA per 128 text rows (latest first), each with its summary
    tiles and text key tiles of 128 from t_lo."""
    assert rows[0] == [nt] and len(rows) == 1 + nt
    coff = offsets([-(-n // k) for n in seqlens])
    covered = {b: [] for b in range(len(seqlens))}
    for r in rows[1:]:
        Q = dict(zip(QT, r))
        b, n = Q["b"], seqlens[Q["b"]]
        assert (Q["n"], Q["m"], Q["c0"]) == (n, n // k, coff[b])
        q0, qn = Q["q0"], Q["qn"]
        assert q0 % BK == 0 and 1 <= qn <= BK and q0 + qn <= n and (qn == BK or q0 + qn == n)
        assert Q["c_first"] == q0 // k
        covered[b].append(q0)
        vt, vs = text_views(n, k, w)
        seen_t = np.flatnonzero(vt[q0:q0 + qn].any(axis=0))
        seen_s = np.flatnonzero(vs[q0:q0 + qn].any(axis=0))
        t_lo, n_win, n_sum = Q["t_lo"], Q["n_win"], Q["n_sum"]
        assert t_lo % k == 0, "a text key box starts on a chunk"
        assert seen_t[0] >= t_lo and seen_t[-1] < t_lo + n_win * BK
        for j in range(n_win):
            assert np.any((seen_t >= t_lo + j * BK) & (seen_t < t_lo + (j + 1) * BK)), ("fully masked text tile", Q, j)
        assert seen_s.size == Q["ns"] and (seen_s.size == 0 or seen_s[-1] == seen_s.size - 1)
        assert n_sum == -(-Q["ns"] // BK)
    for b, n in enumerate(seqlens):
        assert sorted(covered[b]) == list(range(0, n, BK))


@pytest.mark.parametrize("k", [1, 2, 4, 8, 16, 32, 64, 128])   # the tensor-core backward's k: divisors of 128
@pytest.mark.parametrize("w", [0, 1, 3, 8])
def test_backward_key_tiles_and_query_ranges(harness, k, w):
    rng = np.random.default_rng(500 + 10 * k + w)
    lens = [int(x) for x in rng.integers(1, 900 if k > 2 else 350, size=3)] + [0, k, 2 * BK * max(1, k // 8)]
    lens = [min(n, 1400) for n in lens]
    Hq, Hkv = [(32, 8), (8, 8), (64, 4)][(k + w) % 3]
    bwd_case(harness, k, w, Hq, Hkv, lens)


@pytest.mark.parametrize("k,w,G", [(1, 0, 16), (8, 0, 1), (8, 64, 4), (64, 1, 8), (128, 0, 4), (2, 300, 2)])
def test_backward_launch_bounds_at_their_edges(harness, k, w, G):
    """Shapes that push the grid bounds: one long sequence (a summary tile's
    query range is the whole sequence), many short ones (partial tiles per
    sequence), a window wider than the sequence."""
    for lens in ([4000], [1] * 40, [k] * 17 + [k + 1] * 5, [129, 257, 383]):
        bwd_case(harness, k, w, 8 * G, 8, lens)


def _sees(n, k, w, q, kind, key):
    """Text query q sees key (text position or summary index) by the
    oracle's visibility rule; queries outside [0, n) see nothing."""
    return 0 <= q < n and oracle.visible(n, k, w, TEXT, q, kind, key)


def _check_span(n, k, w, kind, first, last, lo, hi):
    """[lo, hi) is exactly the span of text queries that see some key of
    first..last.  Each key's visible queries form one interval; the first
    key's starts earliest.  A text key's interval ends at its chunk's window
    end, latest for the last key; a summary's runs to the end of the
    sequence when it is seen at all, and the first summary is seen if any."""
    if hi <= lo:
        assert not _sees(n, k, w, n - 1, kind, first), "a key seen by the last query got an empty range"
        return
    end_key = last if kind == TEXT else first
    assert 0 <= lo < hi <= n
    assert _sees(n, k, w, lo, kind, first) and not _sees(n, k, w, lo - 1, kind, first)
    assert _sees(n, k, w, hi - 1, kind, end_key) and not _sees(n, k, w, hi, kind, end_key)


@pytest.mark.parametrize("w", [0, 5, (1 << 27) - 1])
def test_backward_ranges_on_a_sequence_of_2_31_tokens(harness, w):
    """One sequence of INT32_MAX tokens (k = 8; w up to the largest accepted
    window): the summary tiles from j0 = 2^27 on, and the text tiles past
    position 2^30, have a window end (j + w + 1) k beyond INT32_MAX.  Each
    tile's query range and the ranges of its key rows are checked against
    the oracle's visibility rule at their ends."""
    k, n = 8, (1 << 31) - 1
    m = n // k
    ns, nt = -(-m // BK), -(-n // BK)
    pick_s = [0, 1, (1 << 27) // BK - 1, (1 << 27) // BK, (1 << 27) // BK + 1, ns - 2, ns - 1]
    pick_t = [0, (1 << 30) // BK - 1, (1 << 30) // BK, nt // 2, nt - 2, nt - 1]
    tiles = pick_s + [ns + t for t in pick_t]
    rows = harness("bwdt", k, w, n, *tiles)
    assert len(rows) == 2 * len(tiles)
    nqs = 64   # k divides 64
    for i, t in enumerate(tiles):
        T = dict(zip(KT, rows[2 * i]))
        kind = SUMMARY if t < ns else TEXT
        j0 = (t if t < ns else t - ns) * BK
        count = m if kind == SUMMARY else n
        kc = min(BK, count - j0)
        assert (T["b"], T["sum"], T["j0"], T["kcnt"], T["n"], T["m"], T["c0"]) == (0, int(kind == SUMMARY), j0, kc, n, m, 0)
        _check_span(n, k, w, kind, j0, j0 + kc - 1, T["qlo"], T["qhi"])
        assert T["nq"] == (-(-(T["qhi"] - T["qlo"]) // nqs) if T["qhi"] > T["qlo"] else 0)
        lohi = rows[2 * i + 1]
        for r, (lo, hi) in zip((0, 1, kc - 1), zip(lohi[0::2], lohi[1::2])):
            _check_span(n, k, w, kind, j0 + r, j0 + r, lo, hi)


# ---------------------------------------------------------------------------
# Decode slice
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("k,w", [(1, 0), (1, 3), (3, 2), (4, 0), (8, 1), (8, 8), (16, 3), (64, 2)])
def test_decode_slice_matches_the_oracle_cache(harness, k, w):
    n_tokens = 40 * k if k <= 8 else 6 * k
    cache = oracle.Cache(k, w, 1, 2, n_tokens // k + 1)
    row = np.zeros((1, 2))
    n = m = 0
    for _ in range(n_tokens):
        assert cache.append_text(row, row) >= 0
        n += 1
        ok, lo, hi = harness("slice", k, w, TEXT, n, m)[0]
        assert ok == 1 and (lo, hi) == cache.slice(TEXT), (n, m)
        assert 1 <= lo < hi <= 1 + k + w * k + m   # within a cache whose capacity is m
        # a summary query is refused while the chunk is incomplete
        assert harness("slice", k, w, SUMMARY, n, m)[0][0] == (1 if n - m * k == 0 and m >= 1 else 0)
        if n % k == 0:
            assert cache.append_summary(row, row) >= 0
            m += 1
            ok, lo, hi = harness("slice", k, w, SUMMARY, n, m)[0]
            assert ok == 1 and (lo, hi) == cache.slice(SUMMARY), (n, m)
            # a text query needs its token in the cache: f = n - m k >= 1
            assert harness("slice", k, w, TEXT, n, m)[0][0] == 0
    assert harness("slice", k, w, SUMMARY, 0, 0)[0][0] == 0
    assert harness("slice", k, w, TEXT, k + 1, 0)[0][0] == 0   # f > k
    # counts no sequence of appends reaches, even where f would pass
    for n_, m_ in ((-k, -2), (1 - k, -1), (-1, 0), (k, -1)):
        assert harness("slice", k, w, TEXT, n_, m_)[0][0] == 0
        assert harness("slice", k, w, SUMMARY, n_, m_)[0][0] == 0


# ---------------------------------------------------------------------------
# Chunked prefill: where each key is read from
# ---------------------------------------------------------------------------
def oracle_cache_image(k, w, n0, m0, cap):
    """The oracle's cache after n0 text appends and m0 summaries (in the
    order of section 2.3.1), each K row holding its key's id: text p -> p + 1,
    summary j -> -(j + 1)."""
    cache = oracle.Cache(k, w, 1, 1, cap)
    m = 0
    for p in range(n0):
        assert cache.append_text(np.full((1, 1), p + 1.0), np.zeros((1, 1))) == 0
        if (p + 1) % k == 0 and m < m0:
            assert cache.append_summary(np.full((1, 1), -(m + 1.0)), np.zeros((1, 1))) == 0
            m += 1
    assert (cache.n_text, cache.m) == (n0, m0)
    return cache.K()[:, 0, 0]


@pytest.mark.parametrize("k,w", [(1, 0), (1, 2), (2, 1), (3, 2), (4, 1), (4, 4), (8, 2), (8, 8), (16, 3), (5, 0)])
def test_chunk_keys_are_read_where_the_cache_holds_them(harness, k, w):
    rng = np.random.default_rng(900 + 10 * k + w)
    states = [(0, 0, 3 * k + 1), (k - 1, 0, 2), (2 * k, 2, k), (3 * k, 2, 1), (3 * k, 2, 2 * k + 3)]
    for _ in range(4):
        n0 = int(rng.integers(0, 12 * k + 5))
        pending = n0 > 0 and n0 % k == 0 and rng.random() < 0.5   # a full chunk still waiting for its summary
        states.append((n0, n0 // k - (1 if pending else 0), int(rng.integers(1, 4 * k + 3))))
    for n0, m0, T in states:
        f0 = n0 - m0 * k
        S_new = (f0 + T) // k
        n1, m1 = n0 + T, m0 + S_new
        img = oracle_cache_image(k, w, n0, m0, m1 + 1)
        where = {}
        for kind, idx, src, at in harness("keys", k, w, n0, m0, T):
            where[(kind, idx)] = (src, at)
        M = oracle.dense_mask(n1, k, w).astype(bool)
        # Eq. (1) positions of text p and summary j, and the rows the block computes
        tpos = lambda p: (p // k) * (k + 1) + p % k
        spos = lambda j: j * (k + 1) + k
        rows = [tpos(p) for p in range(n0, n1)] + [spos(j) for j in range(m0, m1)]
        seen = M[rows].any(axis=0)
        for p in range(n1):
            if not seen[tpos(p)]:
                continue
            src, at = where[(TEXT, p)]
            if p < n0:
                assert src == 0 and img[at] == p + 1, ("cached text key read from the wrong slot", n0, m0, T, p, at)
            else:
                assert (src, at) == (1, p - n0)
        for j in range(m1):
            if not seen[spos(j)]:
                continue
            src, at = where[(SUMMARY, j)]
            if j < m0:
                assert src == 0 and img[at] == -(j + 1), ("cached summary read from the wrong slot", n0, m0, T, j, at)
            else:
                assert (src, at) == (1, j - m0)



def test_wide_window_tile_lists(harness):
    """The sliding chunk number 128 of the benchmarked sweep (a 1024-token
    window at k = 8): a work item's window spans many K/V tiles; forward
    items, chunked-prefill items and backward tiles all stay exact."""
    fwd_case(harness, 8, 128, 32, 8, [3000, 1100, 9])
    chunk_case(harness, 8, 128, 32, 8, [(1500, 187, 700), (2048, 255, 64), (7, 0, 1200)])
    bwd_case(harness, 8, 128, 32, 8, [3000, 1100, 9])


def test_largest_accepted_window(harness):
    """(w + 1) k = 2^30, the largest window the library accepts: the tile
    lists' 32-bit index arithmetic does not wrap (every row sees all of its
    sequence's earlier text and no summary)."""
    w = (1 << 27) - 1
    fwd_case(harness, 8, w, 32, 8, [1000, 300])
    bwd_case(harness, 8, w, 32, 8, [1000, 300])
    chunk_case(harness, 8, w, 32, 8, [(500, 62, 300)])
