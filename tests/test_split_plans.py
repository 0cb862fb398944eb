"""Host-side tests of the decode launches' split planning.

tests/split_harness.cu compiles the library's own planning code for the
host: the KV-cache decode's split count and workspace size
(cache_decode.cu), and the MLA latent decode's shares (mla::plan: a share
count and a share length `per` in slots) with its workspace size
(mla_decode.cu).  The MLA kernels read share s of a sequence's slice as the
slots [lo + s per, min(hi, lo + (s + 1) per)), so the shares must cover
every slice the cache can present for a call's max_text; the kernels
reject a `per` that is not a whole number of their blocks (64 slots on the
tensor-core pair kernel, 32 on the warp-level kernels).  The slice itself
comes from the oracle's cache model (section 2.3.1 and Figure 4 of the
Kwai Summary Attention Technical Report: current chunk, ring of the last C
chunks, summaries of the chunks that left the ring)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "split_harness.cu")
D_C, D_R = 512, 64


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    exe = str(tmp_path_factory.mktemp("split") / "split_harness")
    # PTX only: the kernels are compiled along with the host code, never run
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=compute_100a", "-std=c++17", "-O1",
                           "-o", exe, SRC])
    proc = subprocess.Popen([exe], stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True)

    def query(*words):
        proc.stdin.write(" ".join(str(x) for x in words) + "\n")
        proc.stdin.flush()
        return [int(x) for x in proc.stdout.readline().split()]

    yield query
    proc.stdin.close()
    proc.wait(timeout=30)


def _mla(harness, k, w, H, batch, max_text):
    tc, mt, groups, splits, per, ws = harness("mla", k, w, H, batch, max_text)
    return dict(tc=tc, mt=mt, groups=groups, splits=splits, per=per, ws=ws)


def _check_mla_plan(P, H, batch, need):
    blk = 64 if P["tc"] else 32
    assert P["tc"] == (H % 128 == 0)
    assert P["per"] >= blk and P["per"] % blk == 0
    assert 1 <= P["splits"] <= 1024
    assert P["splits"] * P["per"] >= need              # every live slot has a share
    # the partial rows the share kernels write and the merge reads back:
    # d_c floats of O and (max, sum) per (split, sequence, head)
    assert P["ws"] >= P["splits"] * batch * H * (D_C + 2) * 4


@pytest.mark.parametrize("k,w", [(1, 0), (4, 3), (8, 8), (16, 2), (3, 5)])
def test_mla_shares_cover_every_slice_of_the_cache_model(harness, k, w):
    """Step a one-sequence cache through text appends and summary appends
    (the summary of a full chunk added as the next step, as the decode
    lifecycle does) and check, at every state and for both step kinds, that
    a call with max_text = the tokens so far gets shares covering the
    slice the cache model presents."""
    n_max = k * (w + 40) + 3
    cache = oracle.Cache(k, w, 1, 1, n_max // k + 2)
    one = np.zeros(1)
    for n in range(1, n_max + 1):
        assert cache.append_text(one, one) == 0
        states = [cache.slice(oracle.TEXT), cache.slice(oracle.SUMMARY)]
        if n % k == 0:
            assert cache.append_summary(one, one) == 0
            states.append(cache.slice(oracle.TEXT))
        need = max(hi - lo for lo, hi in states)
        for H in (16, 32, 64, 128, 256):
            _check_mla_plan(_mla(harness, k, w, H, 1, n), H, 1, need)


def _largest_slice(k, w, n):
    """Live slots of a TEXT step at n tokens with all full chunks summarised
    but the last (the cache model's slice, checked against the model itself
    by the test above): up to k tokens of the current chunk, the ring's
    min(m, w) chunks and the m - w summaries outside it."""
    m = n // k
    worst = 0
    for mm in {m, max(m - 1, 0)}:
        fp = n - mm * k
        if fp > k:
            continue
        worst = max(worst, fp + min(mm, w) * k + max(mm - w, 0))
    return worst


@pytest.mark.parametrize("H", [16, 32, 64, 128, 256])
def test_mla_plans_at_long_contexts_and_large_batches(harness, H):
    for k, w in [(8, 8), (1, 0), (64, 15), (2, 1000)]:
        for batch in (0, 1, 3, 16, 64, 300):
            for n in (0, 1, 7, 8, 1000, 32768, 131072, 1 << 20, 1 << 27, (1 << 31) - 1):
                P = _mla(harness, k, w, H, batch, n)
                _check_mla_plan(P, H, batch, _largest_slice(k, w, n))


def test_mla_plans_of_the_benchmarked_shapes(harness):
    """Table 1's MLA shape (128 heads, k 8, w 8) at the sweep's points: one
    share per sequence when 64 sequences already fill the pairs, more and
    shorter shares for fewer sequences."""
    one = [_mla(harness, 8, 8, 128, 64, n)["splits"] for n in (32768, 131072)]
    assert one == [1, 1]
    s16 = _mla(harness, 8, 8, 128, 16, 131072)["splits"]
    s1 = _mla(harness, 8, 8, 128, 1, 131072)["splits"]
    assert 1 < s16 < s1
    # pairs of CTAs per wave = SMs / 2: 16 sequences x s16 shares fit in one wave
    assert 16 * s16 <= 148 // 2


def _dec(harness, k, w, Hq, Hkv, d, batch, max_text):
    s, split_bytes, ws = harness("dec", k, w, Hq, Hkv, d, batch, max_text)
    return s, split_bytes, ws


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (16, 16, 64), (64, 8, 128), (8, 1, 64)])
def test_decode_split_counts_and_workspace(harness, Hq, Hkv, d):
    """1 <= splits <= 1024; each split's partials are (d + 2) floats per
    (sequence, q head) and the workspace holds all splits; more sequences
    never take more splits, a longer context never fewer."""
    for k, w in [(8, 8), (1, 0), (64, 15)]:
        texts = (0, 1, 100, 4096, 32768, 131072, 1 << 20, 1 << 30)
        batches = (1, 2, 16, 64, 128, 1000)
        grid = {}
        for batch in batches:
            for n in texts:
                s, split_bytes, ws = _dec(harness, k, w, Hq, Hkv, d, batch, n)
                assert 1 <= s <= 1024
                assert split_bytes == 4 * batch * Hq * (d + 2)
                assert ws >= s * split_bytes and ws % 16 == 0
                grid[batch, n] = s
        for n in texts:
            col = [grid[b, n] for b in batches]
            assert col == sorted(col, reverse=True), (k, w, n, col)
        for b in batches:
            row = [grid[b, n] for n in texts]
            assert row == sorted(row), (k, w, b, row)
