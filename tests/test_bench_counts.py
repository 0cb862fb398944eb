"""The benchmark's work counts, checked against the oracle.

bench.py reports prefill throughput as FLOPs of the visible (query, key)
pairs and decode bandwidth as bytes of the cache slice, both from closed
forms.  The closed forms are checked here against the dense mask ("Kwai
Summary Attention Technical Report", section 2.2.1 and section 2.2.2,
Eqs. (2)-(3)), the oracle's pair enumeration (whose totals are pinned in
test_oracle_pins.py) and the oracle cache's decode slice (section 2.3.1,
Figure 4).  The tests cover the whole prefill, its text rows, a
chunked-prefill block, and one TEXT decode step.
"""
from __future__ import annotations

import numpy as np
import pytest

import bench
import oracle

TEXT = 0


def mask_views(n, k, w):
    """Dense mask with the Eq. (1) positions of text p and summary j."""
    M = oracle.dense_mask(n, k, w).astype(bool)
    tpos = lambda p: (p // k) * (k + 1) + p % k
    spos = lambda j: j * (k + 1) + k
    return M, tpos, spos


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("w", [0, 1, 2, 7])
def test_useful_and_text_pairs_equal_the_mask(k, w):
    rng = np.random.default_rng(10 * k + w)
    lens = [0, 1, k, k + 1] + [int(x) for x in rng.integers(2, 260, size=3)]
    total = text = 0
    for n in lens:
        M, tpos, _ = mask_views(n, k, w)
        total += int(M.sum())
        text += int(M[[tpos(p) for p in range(n)]].sum())
    assert bench.useful_pairs(lens, k, w) == total
    assert bench.text_pairs(lens, k, w) == text


def test_useful_pairs_of_the_benchmarked_workloads():
    """The 32768-token prefill (k 8, w 8) and the packed 217K-token batch
    (k 8, w 16): the oracle's enumeration, whose totals are pinned."""
    n = bench.PF["seqlens"][0]
    assert bench.useful_pairs([n], bench.PF["k"], bench.PF["w"]) == int(
        oracle.lib().oracle_count_pairs(n, bench.PF["k"], bench.PF["w"])) == 69109792
    lens = (131072, 65536, 16384, 4000)
    assert bench.useful_pairs(lens, 8, 16) == 1385339220


@pytest.mark.parametrize("k,w", [(1, 0), (2, 3), (4, 1), (8, 2), (8, 8), (16, 1)])
def test_chunk_pairs_equal_the_block_rows_of_the_mask(k, w):
    """A block of T tokens after n0 cached ones: its text rows and the
    summary rows of the chunks it completes, on the mask of n0 + T tokens
    (a chunked prefill computes exactly these rows of the prefill)."""
    rng = np.random.default_rng(40 + k + w)
    cases = [(0, 0, 3 * k + 1), (k - 1, 0, 2), (3 * k, 2, 1), (3 * k, 3, k)]
    for _ in range(4):
        n0 = int(rng.integers(0, 10 * k + 3))
        pending = n0 > 0 and n0 % k == 0 and rng.random() < 0.5
        cases.append((n0, n0 // k - (1 if pending else 0), int(rng.integers(1, 5 * k))))
    for n0, m0, T in cases:
        n1 = n0 + T
        M, tpos, spos = mask_views(n1, k, w)
        rows = [tpos(p) for p in range(n0, n1)] + [spos(j) for j in range(m0, n1 // k)]
        assert bench.chunk_pairs(n0, m0, T, k, w) == int(M[rows].sum()), (n0, m0, T)


@pytest.mark.parametrize("k,w", [(1, 0), (1, 3), (4, 2), (8, 8), (16, 1)])
def test_decode_slice_rows_equal_the_oracle_cache(k, w):
    """One TEXT step after m summaries and `fill` open tokens reads the
    slice of the oracle's cache after that step's append, which holds
    exactly the keys the mask gives the new token."""
    row = np.zeros((1, 1))
    for m in (0, 1, w, w + 1, 3 * w + 5):
        for fill in range(k):
            cache = oracle.Cache(k, w, 1, 1, m + 1)
            for p in range(m * k + fill + 1):
                assert cache.append_text(row, row) == 0
                if (p + 1) % k == 0 and cache.m < m:
                    assert cache.append_summary(row, row) == 0
            lo, hi = cache.slice(TEXT)
            n = m * k + fill + 1
            M, tpos, _ = mask_views(n, k, w)
            assert bench.decode_slice_rows(m, k, w, [fill])[0] == hi - lo == int(M[tpos(n - 1)].sum())


@pytest.mark.parametrize("k,w", [(1, 0), (3, 2), (8, 8), (16, 1)])
def test_text_row_keys_row_by_row(k, w):
    """The per-row key count (shared by the pair totals and the CPU
    baseline's FLOP count) equals each text row's mask row."""
    for n in (1, k, 5 * k + 3, 200):
        M, tpos, _ = mask_views(n, k, w)
        want = [int(M[tpos(p)].sum()) for p in range(n)]
        assert bench.text_row_keys(np.arange(n), k, w, n // k).tolist() == want
