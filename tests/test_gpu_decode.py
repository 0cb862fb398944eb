"""GPU parity of ksa_cache_append and ksa_decode (Kwai Summary Attention
Technical Report, section 2.3.1, Figure 4) against the fp64 oracle: the
cache bytes bit for bit against the oracle's slot map, and decode outputs
against the oracle's masked prefill rows and its cache-model decode."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import DecodeCache
from kv_cache_compression_ksa_b200.inputs import fill_normal_, token_stream, uniform_ints
from ksa_testutil import LSE_ABS, RowSet, assert_close, to_f64

pytestmark = pytest.mark.gpu
THETA = 1e6
TEXT, SUMMARY, SKIP = L.KSA_TEXT, L.KSA_SUMMARY, L.KSA_SKIP


def gpu_image(cache: DecodeCache, b: int):
    """[S, Hkv, d] fp64 image of sequence b (library layout is [B, Hkv, S, d])."""
    return to_f64(cache.k[b].transpose(0, 1)), to_f64(cache.v[b].transpose(0, 1))


def test_append_slot_map_bit_exact():
    """RoPE off, so an append is a pure copy: after every step the whole GPU
    cache equals the oracle's slot map byte for byte (current chunk right to
    left, scratch, ring block copy modulo w, summary buffer), including ring
    wrap-around, sequences at different phases, SKIP and error cases."""
    k, w, Hq, Hkv, d, cap = 4, 2, 4, 2, 64, 9
    B = 3
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, 0.0)
    cache = DecodeCache(p, B, cap)
    models = [oracle.Cache(k, w, Hkv, d, cap) for _ in range(B)]
    rng = np.random.default_rng(0)
    starts = [0, 3, 6]            # sequence b starts appending at step starts[b]
    pending = [False] * B         # chunk complete: next step is its summary
    for step in range(60):
        kinds = []
        for b in range(B):
            if step < starts[b]:
                kinds.append(SKIP)
            elif pending[b]:
                kinds.append(SUMMARY)
            else:
                kinds.append(TEXT)
        kn = torch.from_numpy(rng.standard_normal((B, Hkv, d))).to(torch.bfloat16)
        vn = torch.from_numpy(rng.standard_normal((B, Hkv, d))).to(torch.bfloat16)
        kind_t = torch.tensor(kinds, dtype=torch.int8, device="cuda")
        cache.append(kind_t, kn.cuda(), vn.cuda())
        for b in range(B):
            mdl = models[b]
            if kinds[b] == TEXT:
                assert mdl.append_text(to_f64(kn[b]), to_f64(vn[b])) == 0
                pending[b] = (mdl.n_text - mdl.m * k) == k
            elif kinds[b] == SUMMARY:
                rc = mdl.append_summary(to_f64(kn[b]), to_f64(vn[b]))
                if rc == 0:
                    pending[b] = False
                else:
                    assert rc == -3
        torch.cuda.synchronize()
        st = cache.state.cpu().numpy()
        for b in range(B):
            Kg, Vg = gpu_image(cache, b)
            np.testing.assert_array_equal(Kg, models[b].K())
            np.testing.assert_array_equal(Vg, models[b].V())
            assert st[b, 0] == models[b].n_text and st[b, 1] == models[b].m
    # sequence 0 ran out of summary capacity (cap = 9) and recorded it
    assert cache.state[0, 3].item() == L.KSA_ERR_CAPACITY
    # a TEXT append into a complete chunk is an order violation
    errs = cache.state[:, 3].cpu().numpy()
    assert set(errs.tolist()) <= {0, L.KSA_ERR_CAPACITY}


def test_append_order_violation_sets_state_error():
    k, w, Hq, Hkv, d = 2, 1, 2, 1, 64
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, 0.0)
    cache = DecodeCache(p, 1, 4)
    z = torch.zeros(1, Hkv, d, dtype=torch.bfloat16, device="cuda")
    cache.append(torch.tensor([SUMMARY], dtype=torch.int8, device="cuda"), z, z)  # chunk not complete
    torch.cuda.synchronize()
    assert cache.state[0, 3].item() == L.KSA_ERR_STATE
    assert cache.state[0, 0].item() == 0 and cache.state[0, 1].item() == 0


@pytest.mark.parametrize("k,w,Hq,Hkv,d", [(8, 2, 8, 2, 128), (4, 1, 4, 4, 64), (3, 3, 16, 2, 128)])
def test_decode_steps_equal_prefill_rows(k, w, Hq, Hkv, d):
    """Two sequences decode token by token through the cache (RoPE applied
    by the library at the cache's positions).  Text step i equals text row i
    of the oracle's masked prefill; the summary step of chunk j equals
    summary row j (decode == prefill, section 2.3.1)."""
    n = 12 * k + k // 2
    B = 2
    streams = [token_stream(n, k, Hq, Hkv, d, seed=20 + b) for b in range(B)]
    refs = [oracle.ksa_prefill([n], k, w, *[to_f64(t) for t in s], THETA)[0] for s in streams]
    m = n // k
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    cache = DecodeCache(p, B, cap=m + 1)
    ws = cache.workspace(n)
    offset = [0, 5]  # the second sequence starts 5 steps later
    # per-sequence event lists: ('t', i) or ('s', j)
    events = []
    for b in range(B):
        ev = [("skip", None)] * offset[b]
        for i in range(n):
            ev.append(("t", i))
            if (i + 1) % k == 0:
                ev.append(("s", (i + 1) // k - 1))
        events.append(ev)
    steps = max(len(e) for e in events)
    rows = RowSet(f"decode outputs k{k} w{w} G{Hq // Hkv} d{d}")
    for s in range(steps):
        kinds, kn, vn, qn = [], [], [], []
        for b in range(B):
            ev = events[b][s] if s < len(events[b]) else ("skip", None)
            qt, kt, vt, qs, ks, vs = streams[b]
            if ev[0] == "t":
                kinds.append(TEXT); kn.append(kt[ev[1]]); vn.append(vt[ev[1]]); qn.append(qt[ev[1]])
            elif ev[0] == "s":
                kinds.append(SUMMARY); kn.append(ks[ev[1]]); vn.append(vs[ev[1]]); qn.append(qs[ev[1]])
            else:
                kinds.append(SKIP); kn.append(torch.zeros(Hkv, d, dtype=torch.bfloat16))
                vn.append(kn[-1]); qn.append(torch.zeros(Hq, d, dtype=torch.bfloat16))
        kind_t = torch.tensor(kinds, dtype=torch.int8, device="cuda")
        cache.append(kind_t, torch.stack(kn).cuda(), torch.stack(vn).cuda())
        o, lse = cache.decode(kind_t, torch.stack(qn).cuda(), n, ws)
        o, lse = to_f64(o), to_f64(lse)
        for b in range(B):
            ev = events[b][s] if s < len(events[b]) else ("skip", None)
            r = refs[b]
            if ev[0] == "t":
                rows.add(o[b], r.text_o[ev[1]], f"text step {ev[1]}")
                assert_close(lse[b], r.text_lse[ev[1]], f"text lse {ev[1]}", max_abs=LSE_ABS, rel_frob=None)
            elif ev[0] == "s":
                rows.add(o[b], r.sum_o[ev[1]], f"summary step {ev[1]}")
                assert_close(lse[b], r.sum_lse[ev[1]], f"summary lse {ev[1]}", max_abs=LSE_ABS, rel_frob=None)
    rows.check()
    assert (cache.state[:, 3] == 0).all()


def _prefilled_cache(B, k, w, Hq, Hkv, d, m_chunks, fills, seed):
    """A cache whose every slot holds N(0,1) bf16 and whose state says each
    sequence has m_chunks complete chunks plus fills[b] open tokens."""
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    cache = DecodeCache(p, B, cap=m_chunks + 8)
    fill_normal_(cache.k, seed)
    fill_normal_(cache.v, seed + 1)
    st = torch.zeros(B, 4, dtype=torch.int32)
    st[:, 0] = torch.as_tensor(m_chunks * k + np.asarray(fills), dtype=torch.int32)
    st[:, 1] = m_chunks
    cache.state.copy_(st)
    return p, cache


@pytest.mark.parametrize("B,m_chunks,nsample", [(64, 16384, 6), (2, 131072, 2), (3, 40, 3)])
def test_decode_full_size_against_cache_model(B, m_chunks, nsample):
    """The long-context decode step (64 sequences, 16384 summaries each, full
    64-token ring, fill 0..7; and the 1M-token context, 131072 summaries, of
    the decode sweep): one TEXT append + decode in the launch configuration
    the benchmark times, checked on sampled sequences against the oracle's
    cache-model decode of the same cache image."""
    k, w, Hq, Hkv, d = 8, 8, 32, 8, 128
    fills = uniform_ints(B, 0, k - 1, seed=3).numpy()
    p, cache = _prefilled_cache(B, k, w, Hq, Hkv, d, m_chunks, fills, seed=9)
    gen = torch.Generator(device="cuda").manual_seed(4)
    kn = torch.randn(B, Hkv, d, generator=gen, device="cuda").to(torch.bfloat16)
    vn = torch.randn(B, Hkv, d, generator=gen, device="cuda").to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=gen, device="cuda").to(torch.bfloat16)
    kind = torch.zeros(B, dtype=torch.int8, device="cuda")
    max_text = m_chunks * k + k
    cache.append(kind, kn, vn)
    o, lse = cache.decode(kind, q, max_text)
    torch.cuda.synchronize()
    o, lse = to_f64(o), to_f64(lse)
    st = cache.state.cpu().numpy()
    assert np.all(st[:, 3] == 0)
    np.testing.assert_array_equal(st[:, 0], m_chunks * k + fills + 1)
    pos = st[:, 0] - 1
    rows = RowSet(f"decode {B} x {m_chunks} summaries")
    for b in sorted(set(np.linspace(0, B - 1, nsample).astype(int).tolist())):
        Kimg, Vimg = gpu_image(cache, b)
        # the oracle rotates the bf16 input query itself, in fp64
        qr = oracle.rope(to_f64(q[b])[None], np.array([pos[b]]), THETA)[0]
        want_o, want_l = oracle.decode_image(k, w, cache.cap, int(st[b, 0]), int(st[b, 1]), oracle.TEXT,
                                             Kimg, Vimg, qr)
        rows.add(o[b], want_o, f"decode seq {b}")
        assert_close(lse[b], want_l, f"decode lse {b}", max_abs=LSE_ABS, rel_frob=None)
        # the appended key is the rotated input, one bf16 rounding away
        kr = oracle.rope(to_f64(kn[b])[None], np.array([pos[b]]), THETA)[0]
        slot = k - fills[b]
        assert np.all(np.abs(Kimg[slot] - kr) <= 2.0 ** -8 * np.abs(kr) + 1e-5)
    rows.check()


def test_decode_multistep_ring_wrap_and_summaries():
    """64 consecutive steps from a 4K context (16 sequences, w = 8): text
    appends with a summary step whenever a chunk completes, so the ring wraps
    and summaries are appended mid-run.  Every step of two sampled sequences
    is checked against the oracle's decode of the cache image."""
    k, w, Hq, Hkv, d = 8, 8, 32, 8, 128
    B, m0 = 16, 512
    fills = uniform_ints(B, 0, k - 1, seed=7).numpy()
    p, cache = _prefilled_cache(B, k, w, Hq, Hkv, d, m0, fills, seed=70)
    gen = torch.Generator(device="cuda").manual_seed(71)
    ws = cache.workspace(m0 * k + 80)
    fill = fills.copy()
    watch = [0, 11]
    rows = RowSet("decode multistep outputs")
    for step in range(64):
        for phase in ("text", "summary"):
            if phase == "text":
                kinds = np.full(B, TEXT)
            else:
                kinds = np.where(fill == k, SUMMARY, SKIP)
                if not np.any(kinds == SUMMARY):
                    continue
            kind = torch.as_tensor(kinds, dtype=torch.int8, device="cuda")
            kn = torch.randn(B, Hkv, d, generator=gen, device="cuda").to(torch.bfloat16)
            vn = torch.randn(B, Hkv, d, generator=gen, device="cuda").to(torch.bfloat16)
            q = torch.randn(B, Hq, d, generator=gen, device="cuda").to(torch.bfloat16)
            cache.append(kind, kn, vn)
            o, lse = cache.decode(kind, q, m0 * k + 80, ws)
            torch.cuda.synchronize()
            st = cache.state.cpu().numpy()
            for b in watch:
                if kinds[b] == SKIP:
                    continue
                Kimg, Vimg = gpu_image(cache, b)
                qr = oracle.rope(to_f64(q[b])[None], np.array([st[b, 0] - 1]), THETA)[0]
                kd = oracle.TEXT if kinds[b] == TEXT else oracle.SUMMARY
                want_o, want_l = oracle.decode_image(k, w, cache.cap, int(st[b, 0]), int(st[b, 1]), kd,
                                                     Kimg, Vimg, qr)
                rows.add(to_f64(o[b]), want_o, f"step {step} seq {b} {phase}")
                assert_close(to_f64(lse[b]), want_l, f"step {step} seq {b} lse", max_abs=LSE_ABS, rel_frob=None)
            if phase == "text":
                fill = fill + 1
            else:
                fill = np.where(kinds == SUMMARY, 0, fill)
    rows.check()
    assert (cache.state[:, 3] == 0).all()
    assert (cache.state[:, 1].cpu().numpy() > m0).all()
