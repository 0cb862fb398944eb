"""ksa_decode_noalloc: the decode step for callers that cannot allocate
device memory (a host program that owns all of the GPU's memory, or a custom
op handed only its inputs and outputs).  It must give the same results as
ksa_decode with a caller-provided workspace, call after call, although its
scratch is one fixed array the library keeps for the life of the process
(and may therefore run fewer split-K splits), and match the oracle.

This file is collected last on purpose, so that a stop-at-first-failure run
has already run every other test if this one fails."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import DecodeCache
from kv_cache_compression_ksa_b200.inputs import fill_normal_, uniform_ints
from ksa_testutil import LSE_ABS, MAX_ABS, RowSet, assert_close, to_f64

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 4 << 20  # bytes the library documents for the fixed scratch


def _cache(B, m, k=8, w=8, Hq=32, Hkv=8, d=128, seed=40):
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, 1e6)
    cache = DecodeCache(p, B, cap=m + 8)
    fill_normal_(cache.k, seed)
    fill_normal_(cache.v, seed + 1)
    fills = uniform_ints(B, 0, k - 1, seed=seed + 2).numpy()
    st = torch.zeros(B, 4, dtype=torch.int32)
    st[:, 0] = torch.as_tensor(m * k + fills, dtype=torch.int32)
    st[:, 1] = m
    cache.state.copy_(st)
    return p, cache


def _two_calls(p, cache, kind, max_text, seed, stream=None):
    """Two decode calls in a row through both entry points, each on the
    same fresh queries; returns the queries and both results per call."""
    gen = torch.Generator(device="cuda").manual_seed(seed)
    out = []
    for call in range(2):
        q = torch.randn(cache.batch, p.num_q_heads, p.head_dim, generator=gen, device="cuda").to(torch.bfloat16)
        o1, l1 = cache.decode(kind, q, max_text, stream=stream)         # caller-provided workspace
        o2 = torch.full_like(o1, float("nan"))
        l2 = torch.full_like(l1, float("nan"))
        L.ksa_decode_noalloc(p, cache.desc, kind, q, o2, l2, max_text, stream=stream)
        out.append((q, o1, l1, o2, l2))
    if stream is None:
        torch.cuda.synchronize()
    else:
        stream.synchronize()
    return [tuple(x if i == 0 else to_f64(x) for i, x in enumerate(t)) for t in out]


def test_noalloc_decode_at_the_benchmark_shape():
    """The benchmarked decode step (64 sequences x 16384 summaries, a full
    64-token ring, 32 q / 8 kv heads, d 128): its split-K partials take more
    than the fixed scratch at ksa_decode's split count, so the call runs
    fewer splits.  Two calls in a row match ksa_decode with a workspace, and
    sampled sequences match the oracle's decode of the cache image."""
    B, m = 64, 16384
    p, cache = _cache(B, m)
    kind = torch.zeros(B, dtype=torch.int8, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(42)
    kn = torch.randn(B, p.num_kv_heads, p.head_dim, generator=gen, device="cuda").to(torch.bfloat16)
    cache.append(kind, kn, kn)
    max_text = m * p.k + p.k
    assert L.ksa_decode_workspace_size(p, B, max_text) > SCRATCH_LIMIT
    results = _two_calls(p, cache, kind, max_text, seed=43)
    st = cache.state.cpu().numpy()
    assert np.all(st[:, 3] == 0)
    rows = RowSet("noalloc decode vs oracle")
    imgs = {b: (to_f64(cache.k[b].transpose(0, 1)), to_f64(cache.v[b].transpose(0, 1))) for b in (0, 31, 63)}
    for call, (q, o1, l1, o2, l2) in enumerate(results):
        assert_close(o2, o1, f"noalloc call {call} O vs ksa_decode", max_abs=MAX_ABS)
        assert_close(l2, l1, f"noalloc call {call} LSE vs ksa_decode", max_abs=LSE_ABS, rel_frob=None)
        for b, (Kimg, Vimg) in imgs.items():
            qr = oracle.rope(to_f64(q[b])[None], np.array([st[b, 0] - 1]), 1e6)[0]
            want_o, want_l = oracle.decode_image(p.k, p.w, cache.cap, int(st[b, 0]), int(st[b, 1]), oracle.TEXT,
                                                 Kimg, Vimg, qr)
            rows.add(o2[b], want_o, f"noalloc call {call} seq {b}")
            assert_close(l2[b], want_l, f"noalloc call {call} seq {b} LSE", max_abs=LSE_ABS, rel_frob=None)
    rows.check()
    # the two calls used different queries: the second result is not a stale copy
    assert not np.array_equal(results[0][3], results[1][3])


@pytest.mark.parametrize("G,d", [(1, 128), (8, 128), (4, 64)])
def test_noalloc_decode_matches_workspace_decode_twice(G, d):
    """Other head groupings and head sizes, with chunk-boundary and mid-chunk
    sequences in one batch (fills 0..7 before the appended token)."""
    B, m, Hkv = 16, 300, 4
    p, cache = _cache(B, m, Hq=G * Hkv, Hkv=Hkv, d=d, seed=50 + G)
    kind = torch.zeros(B, dtype=torch.int8, device="cuda")
    kn = torch.randn(B, Hkv, d, device="cuda").to(torch.bfloat16)
    cache.append(kind, kn, kn)
    max_text = m * p.k + p.k
    for call, (q, o1, l1, o2, l2) in enumerate(_two_calls(p, cache, kind, max_text, seed=51)):
        assert_close(o2, o1, f"noalloc G{G} d{d} call {call} O", max_abs=MAX_ABS)
        assert_close(l2, l1, f"noalloc G{G} d{d} call {call} LSE", max_abs=LSE_ABS, rel_frob=None)
    assert (cache.state[:, 3] == 0).all()


def test_noalloc_decode_on_a_caller_stream():
    """Both entry points on a stream the caller created give the same result."""
    B, m = 8, 200
    p, cache = _cache(B, m, seed=60)
    kind = torch.zeros(B, dtype=torch.int8, device="cuda")
    kn = torch.randn(B, p.num_kv_heads, p.head_dim, device="cuda").to(torch.bfloat16)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        cache.append(kind, kn, kn, stream=s)      # every sequence gets its open token
        results = _two_calls(p, cache, kind, m * p.k + p.k, seed=61, stream=s)
    assert (cache.state[:, 3] == 0).all()
    for call, (q, o1, l1, o2, l2) in enumerate(results):
        assert_close(o2, o1, f"noalloc on a stream, call {call} O", max_abs=MAX_ABS)
        assert_close(l2, l1, f"noalloc on a stream, call {call} LSE", max_abs=LSE_ABS, rel_frob=None)


def test_noalloc_decode_rejects_problems_beyond_its_scratch():
    """A batch whose single split of partials exceeds the fixed scratch is
    refused with KSA_ERR_CAPACITY before anything is launched."""
    B, m = 2048, 4
    p = L.make_params(8, 8, 32, 8, 128, 0.0, 1e6)
    max_text = 1 << 20
    assert B * 32 * (128 + 2) * 4 > SCRATCH_LIMIT    # one split's partials
    kv = torch.zeros(B, 8, L.ksa_cache_slots(p, m), 128, dtype=torch.bfloat16, device="cuda")
    state = torch.zeros(B, 4, dtype=torch.int32, device="cuda")
    desc = L.make_cache(kv, kv, state, m)
    kind = torch.zeros(B, dtype=torch.int8, device="cuda")
    q = torch.zeros(B, 32, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.full((B, 32, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.KsaError) as e:
        L.ksa_decode_noalloc(p, desc, kind, q, o, None, max_text)
    assert e.value.status == L.KSA_ERR_CAPACITY
    assert torch.all(o == 3.0)
