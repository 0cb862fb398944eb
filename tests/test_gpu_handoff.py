"""GPU parity of ksa_cache_from_prefill (the prefill -> decode hand-off; the
decode cache of Kwai Summary Attention Technical Report section 2.3.1,
Figure 4): the cache built in one pass from a prefill's rotated augmented
K/V equals, slot for slot, the oracle's cache model fed the same rows in
append order, and the decode step after it equals the oracle's prefill row."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import DecodeCache
from kv_cache_compression_ksa_b200.inputs import token_stream
from ksa_testutil import LSE_ABS, RowSet, assert_close, to_f64

pytestmark = pytest.mark.gpu
THETA = 1e6


def _defined_slots(k, w, n):
    """Slots a decode can read after n appended text tokens (and their
    summaries): the open chunk, the ring blocks of the last min(m, w)
    complete chunks, the summary buffer."""
    m, f = n // k, n - (n // k) * k
    s = [k - r for r in range(f)]
    for c in range(max(0, m - w), m):
        s += [k + 1 + (c % w) * k + i for i in range(k)] if w > 0 else []
    s += [1 + k + w * k + j for j in range(m)]
    return np.asarray(sorted(s), dtype=np.int64)


@pytest.mark.parametrize("seqlens,k,w,Hq,Hkv,d", [
    ([37, 8, 100, 3, 0], 4, 2, 4, 2, 64),       # m < w, m >= w, partial chunks, an empty sequence
    ([1000, 2051], 8, 8, 32, 8, 128),           # the bench shape, ring wrapped many times
    ([77, 64], 8, 0, 8, 8, 64),                 # w = 0: no raw-text window
    ([130, 45], 16, 3, 8, 2, 128),              # k = 16
])
def test_cache_from_prefill_equals_appends(seqlens, k, w, Hq, Hkv, d):
    B = len(seqlens)
    streams = [token_stream(n + 1, k, Hq, Hkv, d, seed=40 + b) for b, n in enumerate(seqlens)]
    # the prefill covers the first n tokens of each stream and their summaries
    cat = lambda i, cnt: torch.cat([s[i][:c] for s, c in zip(streams, cnt)]).cuda()
    nt = sum(seqlens)
    ms = [n // k for n in seqlens]
    qt, kt, vt = cat(0, seqlens), cat(1, seqlens), cat(2, seqlens)
    qs, ks, vs = cat(3, ms), cat(4, ms), cat(5, ms)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(seqlens)]), dtype=torch.int32, device="cuda")
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    rows = L.ksa_aug_rows(p, seqlens)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device="cuda")
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device="cuda")
    va = torch.empty_like(ka)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, B, nt), dtype=torch.uint8, device="cuda")
    L.ksa_interleave_rope(p, cu, nt, sum(ms), rows, qt, kt, vt, qs, ks, vs, qa, ka, va, ws)
    cap = max(ms) + 2
    cache = DecodeCache(p, B, cap)
    cache.from_prefill(cu, nt, ka, va, ws)
    torch.cuda.synchronize()
    assert L.ksa_get_device_error(ws) == 0
    st = cache.state.cpu().numpy()
    Ka, Va = to_f64(ka), to_f64(va)
    coff = np.concatenate([[0], np.cumsum([(n + k - 1) // k for n in seqlens])])
    for b, n in enumerate(seqlens):
        m = n // k
        assert tuple(st[b]) == (n, m, 0, 0)
        mdl = oracle.Cache(k, w, Hkv, d, cap)
        for i in range(n):
            r = (coff[b] + i // k) * (k + 1) + i % k
            assert mdl.append_text(Ka[r], Va[r]) == 0
            if (i + 1) % k == 0:
                srow = (coff[b] + i // k) * (k + 1) + k
                assert mdl.append_summary(Ka[srow], Va[srow]) == 0
        slots = _defined_slots(k, w, n)
        Kg = to_f64(cache.k[b].transpose(0, 1))
        Vg = to_f64(cache.v[b].transpose(0, 1))
        np.testing.assert_array_equal(Kg[slots], mdl.K()[slots])
        np.testing.assert_array_equal(Vg[slots], mdl.V()[slots])
    # decoding token n of every sequence after the hand-off equals text row n
    # of the oracle's prefill of n + 1 tokens
    kind = torch.full((B,), L.KSA_TEXT, dtype=torch.int8, device="cuda")
    kn = torch.stack([s[1][n] for s, n in zip(streams, seqlens)]).cuda()
    vn = torch.stack([s[2][n] for s, n in zip(streams, seqlens)]).cuda()
    qn = torch.stack([s[0][n] for s, n in zip(streams, seqlens)]).cuda()
    cache.append(kind, kn, vn)
    o, lse = cache.decode(kind, qn, max(seqlens) + 1)
    o, lse = to_f64(o), to_f64(lse)
    assert (cache.state[:, 3] == 0).all()
    rows = RowSet("decode after hand-off")
    for b, n in enumerate(seqlens):
        s = streams[b]
        ref = oracle.ksa_prefill([n + 1], k, w, *[to_f64(t) for t in s], THETA, text_rows=[np.array([n])],
                                 sum_rows=[np.zeros(0, np.int64)])[0]
        rows.add(o[b], ref.text_o[0], f"decode after hand-off, seq {b}")
        assert_close(lse[b], ref.text_lse[0], f"lse after hand-off, seq {b}", max_abs=LSE_ABS, rel_frob=None)
    rows.check()


def test_cache_from_prefill_capacity_error():
    """A sequence whose summaries exceed the cache's capacity is left
    unwritten and flagged; the others are built."""
    k, w, Hq, Hkv, d = 4, 2, 4, 2, 64
    seqlens = [40, 8]
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    rows = L.ksa_aug_rows(p, seqlens)
    ka = torch.randn(rows, Hkv, d, device="cuda").to(torch.bfloat16)
    va = torch.randn(rows, Hkv, d, device="cuda").to(torch.bfloat16)
    cu = torch.tensor([0, 40, 48], dtype=torch.int32, device="cuda")
    ws = torch.empty(L.ksa_prefill_workspace_size(p, 2, 48), dtype=torch.uint8, device="cuda")
    cache = DecodeCache(p, 2, cap=5)   # sequence 0 has 10 summaries
    cache.from_prefill(cu, 48, ka, va, ws)
    torch.cuda.synchronize()
    st = cache.state.cpu().numpy()
    assert st[0, 3] == L.KSA_ERR_CAPACITY and st[0, 0] == 0
    assert tuple(st[1]) == (8, 2, 0, 0)
