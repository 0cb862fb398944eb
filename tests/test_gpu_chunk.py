"""GPU parity of ksa_prefill_chunk (chunked prefill against the decode cache
of Kwai Summary Attention Technical Report section 2.3.1, Figure 4).

A block of new tokens per sequence is attended against a cache that holds
the sequence's first n0 tokens; its rows must equal the oracle's prefill
rows n0 .. n0+T-1 (and the summaries of the chunks the block completes),
and afterwards the cache must hold, in every slot a decode reads, what the
oracle's cache model holds after appending the same tokens one by one.
Shapes the tensor-core prefill kernel takes run its text rows there (summary
tiles straight from the cache); the 3-heads-per-kv-head case runs them on
the warp-level kernel."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import DecodeCache
from kv_cache_compression_ksa_b200.inputs import token_stream
from ksa_testutil import LSE_ABS, RowSet, assert_close, sample_rows, to_f64

pytestmark = pytest.mark.gpu
THETA = 1e6


def _defined_slots(k, w, n):
    """Slots a decode reads after n text tokens and floor(n/k) summaries."""
    m, f = n // k, n - (n // k) * k
    s = [k - r for r in range(f)]
    if w > 0:
        for c in range(max(0, m - w), m):
            s += [k + 1 + (c % w) * k + i for i in range(k)]
    s += [1 + k + w * k + j for j in range(m)]
    return np.asarray(sorted(s), dtype=np.int64)


def _prefix_cache(p, streams, n0s, pend, cap):
    """A cache holding the first n0 tokens of each stream: the one-pass
    hand-off of the first n0 (or n0 - 1 when the last chunk's summary is to
    be pending) tokens, then one TEXT append for the pending sequences."""
    k, Hq, Hkv, d = p.k, p.num_q_heads, p.num_kv_heads, p.head_dim
    B = len(streams)
    pre = [n - 1 if pd else n for n, pd in zip(n0s, pend)]
    ms = [n // k for n in pre]
    cat = lambda i, cnt: torch.cat([s[i][:c] for s, c in zip(streams, cnt)]).cuda()
    nt = sum(pre)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(pre)]), dtype=torch.int32, device="cuda")
    rows = L.ksa_aug_rows(p, pre)
    qa = torch.empty(max(rows, 1), Hq, d, dtype=torch.bfloat16, device="cuda")
    ka = torch.empty(max(rows, 1), Hkv, d, dtype=torch.bfloat16, device="cuda")
    va = torch.empty_like(ka)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, B, nt), dtype=torch.uint8, device="cuda")
    L.ksa_interleave_rope(p, cu, nt, sum(ms), rows, cat(0, pre), cat(1, pre), cat(2, pre), cat(3, ms), cat(4, ms),
                          cat(5, ms), qa, ka, va, ws)
    cache = DecodeCache(p, B, cap)
    cache.from_prefill(cu, nt, ka, va, ws)
    if any(pend):
        kind = torch.tensor([L.KSA_TEXT if pd else L.KSA_SKIP for pd in pend], dtype=torch.int8, device="cuda")
        kn = torch.stack([s[1][n - 1] if pd else s[1][0] for s, n, pd in zip(streams, n0s, pend)]).cuda()
        vn = torch.stack([s[2][n - 1] if pd else s[2][0] for s, n, pd in zip(streams, n0s, pend)]).cuda()
        cache.append(kind, kn, vn)
    torch.cuda.synchronize()
    assert L.ksa_get_device_error(ws) == 0
    return cache


def _block_inputs(streams, n0s, m0s, Ts, k):
    """The block's text rows n0 .. n0+T-1 and summary rows m0 .. m1-1 of each
    stream, packed by sequence, with their cu arrays."""
    Ss = [(n0 + T) // k - m0 for n0, m0, T in zip(n0s, m0s, Ts)]
    tx = [[s[i][n0:n0 + T] for s, n0, T in zip(streams, n0s, Ts)] for i in range(3)]
    sm = [[s[3 + i][m0:m0 + S] for s, m0, S in zip(streams, m0s, Ss)] for i in range(3)]
    cu_t = torch.tensor(np.concatenate([[0], np.cumsum(Ts)]), dtype=torch.int32, device="cuda")
    cu_s = torch.tensor(np.concatenate([[0], np.cumsum(Ss)]), dtype=torch.int32, device="cuda")
    tx = [torch.cat(x).cuda() for x in tx]
    sm = [torch.cat(x).cuda() for x in sm]
    return Ss, cu_t, cu_s, tx, sm


CASES = {
    # seqs: (n0, pending, T) -- pending: chunk n0/k - 1 complete, summary to come
    "k4_w2_mixed": (4, 2, 4, 2, 64, [(0, False, 37), (20, False, 5), (16, True, 9), (33, False, 0),
                                     (50, False, 64)]),
    "k8_w8_bench_heads": (8, 8, 32, 8, 128, [(2000, False, 300), (517, False, 1000), (0, False, 129)]),
    "w0": (8, 0, 8, 8, 64, [(77, False, 50), (64, True, 0), (5, False, 3)]),
    "k16_w3_gqa4": (16, 3, 8, 2, 128, [(130, False, 200), (45, False, 3), (160, True, 40)]),
    "k1_gqa4": (1, 2, 4, 1, 64, [(10, False, 10), (0, False, 7)]),
    "gqa8": (8, 4, 16, 2, 128, [(300, False, 257), (64, True, 64)]),
    # 3 q heads per kv head: not a tensor-core prefill shape, the text rows
    # take the warp-level kernel
    "gqa3_warp_path": (4, 2, 6, 2, 64, [(37, False, 50), (16, True, 5), (0, False, 9)]),
    # k 32 with 8 q heads per kv head: each kv head's heads split over 2 tiles
    "k32_gqa8_head_split": (32, 2, 16, 2, 128, [(100, False, 300), (64, True, 70)]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_chunk_matches_oracle(name):
    k, w, Hq, Hkv, d, seqs = CASES[name]
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    B = len(seqs)
    n0s = [s[0] for s in seqs]
    pend = [s[1] for s in seqs]
    Ts = [s[2] for s in seqs]
    m0s = [n // k - (1 if pd else 0) for n, pd in zip(n0s, pend)]
    streams = [token_stream(n0 + T + 1, k, Hq, Hkv, d, seed=70 + b) for b, (n0, _, T) in enumerate(seqs)]
    cap = max((n0 + T) // k for n0, _, T in seqs) + 2
    cache = _prefix_cache(p, streams, n0s, pend, cap)
    st0 = cache.state.cpu().numpy()
    for b in range(B):
        assert tuple(st0[b]) == (n0s[b], m0s[b], 0, 0)
    Ss, cu_t, cu_s, tx, sm = _block_inputs(streams, n0s, m0s, Ts, k)
    ws = cache.chunk_workspace(sum(Ts), sum(Ss))
    o_t, o_s, l_t, l_s = cache.prefill_chunk(cu_t, sum(Ts), cu_s, sum(Ss), *tx, *sm, ws=ws)
    torch.cuda.synchronize()
    assert L.ksa_get_device_error(ws) == 0
    st = cache.state.cpu().numpy()
    o_t, o_s, l_t, l_s = to_f64(o_t), to_f64(o_s), to_f64(l_t), to_f64(l_s)
    t0 = s0 = 0
    for b in range(B):
        n0, m0, T, S = n0s[b], m0s[b], Ts[b], Ss[b]
        n1, m1 = n0 + T, m0 + S
        assert tuple(st[b]) == (n1, m1, 0, 0), (b, st[b])
        s = [to_f64(x) for x in streams[b]]
        ref = oracle.ksa_prefill_chunk(n0, m0, T, k, w, *s, THETA)
        if T:
            assert_close(o_t[t0:t0 + T], ref.text_o, f"{name} seq {b} text rows")
            assert_close(l_t[t0:t0 + T], ref.text_lse, f"{name} seq {b} text lse", max_abs=LSE_ABS, rel_frob=None)
        if S:
            assert_close(o_s[s0:s0 + S], ref.sum_o, f"{name} seq {b} summary rows")
            assert_close(l_s[s0:s0 + S], ref.sum_lse, f"{name} seq {b} summary lse", max_abs=LSE_ABS,
                         rel_frob=None)
        # the cache after the block: V slots exactly (a copy), K slots to the
        # rounding of one rotation, against the oracle's cache model fed the
        # same tokens one by one
        pt, ps = oracle.text_positions(n1), oracle.summary_positions(n1, k)
        rk = oracle.rope(s[1][:n1], pt, THETA)
        sk = oracle.rope(s[4][:m1], ps, THETA) if m1 else s[4][:0]
        mdl = oracle.Cache(k, w, Hkv, d, cap)
        for i in range(n1):
            assert mdl.append_text(rk[i], s[2][i]) == 0
            if (i + 1) % k == 0:
                assert mdl.append_summary(sk[(i + 1) // k - 1], s[5][(i + 1) // k - 1]) == 0
        slots = _defined_slots(k, w, n1)
        Kg = to_f64(cache.k[b].transpose(0, 1))[slots]
        Vg = to_f64(cache.v[b].transpose(0, 1))[slots]
        np.testing.assert_array_equal(Vg, mdl.V()[slots])
        assert np.abs(Kg - mdl.K()[slots]).max(initial=0.0) <= 0.02 * max(1.0, np.abs(mdl.K()).max())
        t0 += T
        s0 += S


@pytest.mark.parametrize("k,w,Hq,Hkv,d", [(8, 8, 32, 8, 128), (4, 3, 4, 2, 64)])
def test_chunk_cache_equals_one_pass_handoff(k, w, Hq, Hkv, d):
    """Two blocks through ksa_prefill_chunk leave, in every slot a decode
    reads, the same bits as the one-pass hand-off of the whole sequence
    (both rotate keys with the same routine), and a decode step after them
    matches the oracle's prefill row."""
    seqs = [(0, 700), (300, 333)]
    B = len(seqs)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    n1s = [a + b for a, b in seqs]
    streams = [token_stream(n + 1, k, Hq, Hkv, d, seed=90 + b) for b, n in enumerate(n1s)]
    cap = max(n1s) // k + 2
    cache = DecodeCache(p, B, cap)
    done = [0] * B
    for blk in range(2):
        Ts = [seqs[b][blk] for b in range(B)]
        m0s = [n // k for n in done]
        Ss, cu_t, cu_s, tx, sm = _block_inputs(streams, done, m0s, Ts, k)
        cache.prefill_chunk(cu_t, sum(Ts), cu_s, sum(Ss), *tx, *sm, want_lse=False)
        done = [a + b for a, b in zip(done, Ts)]
    torch.cuda.synchronize()
    assert (cache.state[:, 3] == 0).all()
    # the one-pass hand-off of the same tokens
    ref_cache = _prefix_cache(p, streams, n1s, [False] * B, cap)
    for b, n in enumerate(n1s):
        slots = torch.as_tensor(_defined_slots(k, w, n), device="cuda")
        assert torch.equal(cache.k[b][:, slots], ref_cache.k[b][:, slots])
        assert torch.equal(cache.v[b][:, slots], ref_cache.v[b][:, slots])
    assert torch.equal(cache.state, ref_cache.state)
    kind = torch.full((B,), L.KSA_TEXT, dtype=torch.int8, device="cuda")
    cache.append(kind, torch.stack([s[1][n] for s, n in zip(streams, n1s)]).cuda(),
                 torch.stack([s[2][n] for s, n in zip(streams, n1s)]).cuda())
    o, lse = cache.decode(kind, torch.stack([s[0][n] for s, n in zip(streams, n1s)]).cuda(), max(n1s) + 1)
    o, lse = to_f64(o), to_f64(lse)
    rows = RowSet("decode after chunks")
    for b, n in enumerate(n1s):
        ref = oracle.ksa_prefill([n + 1], k, w, *[to_f64(t) for t in streams[b]], THETA,
                                 text_rows=[np.array([n])], sum_rows=[np.zeros(0, np.int64)])[0]
        rows.add(o[b], ref.text_o[0], f"decode after chunks, seq {b}")
        assert_close(lse[b], ref.text_lse[0], f"lse after chunks, seq {b}", max_abs=LSE_ABS, rel_frob=None)
    rows.check()


def test_chunk_state_errors():
    """A sequence whose block brings the wrong number of summaries, or more
    than the capacity holds, is flagged and left untouched; the others are
    processed."""
    k, w, Hq, Hkv, d = 4, 2, 4, 2, 64
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    streams = [token_stream(64, k, Hq, Hkv, d, seed=120 + b) for b in range(3)]
    cache = _prefix_cache(p, streams, [6, 6, 6], [False] * 3, cap=5)
    # seq 0: fine (6 + 10 -> 4 summaries); seq 1: claims 1 summary instead of
    # 4; seq 2: 6 + 18 tokens -> 6 summaries > cap 5
    Ts = [10, 10, 18]
    Ss = [4 - 1, 1, 6 - 1]
    cu_t = torch.tensor(np.concatenate([[0], np.cumsum(Ts)]), dtype=torch.int32, device="cuda")
    cu_s = torch.tensor(np.concatenate([[0], np.cumsum(Ss)]), dtype=torch.int32, device="cuda")
    tx = [torch.cat([s[i][6:6 + T] for s, T in zip(streams, Ts)]).cuda() for i in range(3)]
    sm = [torch.cat([s[3 + i][1:1 + S] for s, S in zip(streams, Ss)]).cuda() for i in range(3)]
    k_before = cache.k.clone()
    o_t, o_s, _, _ = cache.prefill_chunk(cu_t, sum(Ts), cu_s, sum(Ss), *tx, *sm)
    torch.cuda.synchronize()
    st = cache.state.cpu().numpy()
    assert tuple(st[0]) == (16, 4, 0, 0)
    assert tuple(st[1]) == (6, 1, 0, L.KSA_ERR_STATE)
    assert tuple(st[2]) == (6, 1, 0, L.KSA_ERR_CAPACITY)
    assert torch.equal(cache.k[1:], k_before[1:])
    ref = oracle.ksa_prefill_chunk(6, 1, 10, k, w, *[to_f64(x) for x in streams[0]], THETA)
    assert_close(to_f64(o_t[:10]), ref.text_o, "valid sequence beside failing ones")


def test_chunk_host_errors():
    p = L.make_params(4, 2, 4, 2, 64, 0.0, THETA)
    cache = DecodeCache(p, 2, 4)
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    x = torch.zeros(4, 4, 64, dtype=torch.bfloat16, device="cuda")
    kx = torch.zeros(4, 2, 64, dtype=torch.bfloat16, device="cuda")
    ws = cache.chunk_workspace(4, 0)
    with pytest.raises(L.KsaError) as e:   # text inputs missing
        L.ksa_prefill_chunk(p, cache.desc, cu, 4, cu, 0, None, None, None, None, None, None, x, None, None, None, ws)
    assert e.value.status == L.KSA_ERR_INVALID
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(L.KsaError) as e:
        L.ksa_prefill_chunk(p, cache.desc, cu, 4, cu, 0, x, kx, kx, None, None, None, x, None, None,
                            None, small)
    assert e.value.status == L.KSA_ERR_WORKSPACE
    # cu totals that disagree with the host totals: device error, nothing written
    cu_bad = torch.tensor([0, 2, 3], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.ksa_prefill_chunk(p, cache.desc, cu_bad, 4, cu, 0, x, kx, kx, None, None, None, x, None, None,
                        None, ws, dev_err=err)
    assert L.ksa_get_device_error(err) == L.KSA_ERR_INVALID
    assert (cache.state == 0).all()


def test_chunk_full_size_128k_sampled():
    """A 4096-token block onto a 127K-token cache (32 q / 8 kv heads, d 128,
    k 8, w 8; 15872 summaries already cached): sampled rows against the
    oracle."""
    k, w, Hq, Hkv, d = 8, 8, 32, 8, 128
    n0, T = 131072 - 4096, 4096
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    streams = [token_stream(n0 + T, k, Hq, Hkv, d, seed=5, scale=0.5, device="cuda")]
    cache = _prefix_cache(p, streams, [n0], [False], cap=(n0 + T) // k + 1)
    m0 = n0 // k
    Ss, cu_t, cu_s, tx, sm = _block_inputs(streams, [n0], [m0], [T], k)
    o_t, o_s, l_t, l_s = cache.prefill_chunk(cu_t, T, cu_s, Ss[0], *tx, *sm)
    torch.cuda.synchronize()
    assert (cache.state[:, 3] == 0).all()
    rows = sample_rows(T, 24, seed=3)
    srows = sample_rows(Ss[0], 6, seed=4)
    s = [to_f64(x) for x in streams[0]]
    ref = oracle.ksa_prefill([n0 + T], k, w, *s, THETA, text_rows=[n0 + rows], sum_rows=[m0 + srows])[0]
    assert_close(to_f64(o_t)[rows], ref.text_o, "128K chunk text rows")
    assert_close(to_f64(l_t)[rows], ref.text_lse, "128K chunk lse", max_abs=LSE_ABS, rel_frob=None)
    assert_close(to_f64(o_s)[srows], ref.sum_o, "128K chunk summary rows")
