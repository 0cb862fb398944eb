"""GPU parity of the decode sweep workload: 64 consecutive decode steps per
sequence with cache maintenance, at the sweep's batch x context points
(Kwai Summary Attention Technical Report, section 2.3.1 and Figure 4b-4e:
text write, summary scratch, ring copy, summary append).

The schedule is the one the benchmark's decode sweep times: at every step a
sequence whose open chunk is full takes a SUMMARY step (the append copies
the chunk into the ring, overwriting its oldest block, and appends the
summary), every other sequence a TEXT step; 64 TEXT steps and the 8 SUMMARY
steps they trigger per sequence, through ksa_cache_append and ksa_decode.
Every step of a few watched sequences is compared with the oracle's decode
of the GPU cache image of that step."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import DecodeCache
from kv_cache_compression_ksa_b200.inputs import fill_normal_, uniform_ints
from ksa_testutil import LSE_ABS, RowSet, assert_close, to_f64

pytestmark = pytest.mark.gpu
THETA = 1e6
K, W, HQ, HKV, D = 8, 8, 32, 8, 128
TEXT_STEPS = 64

# (batch, prior context in text tokens, watched sequences)
POINTS = [
    (1, 4096, [0]),
    (128, 32768, [0, 77, 127]),
    (16, 131072, [0, 9, 15]),
    (16, 1048576, [0, 15]),
]


def _schedule(fills, m):
    """Per step and sequence: SUMMARY (1) when the open chunk is full, else
    TEXT (0); a whole number of k+1-step cycles, so every sequence makes 64
    text steps and 8 summary steps whatever its starting fill."""
    nsteps = TEXT_STEPS // K * (K + 1)
    B = len(fills)
    kinds = np.zeros((nsteps, B), np.int8)
    f = fills.copy()
    for j in range(nsteps):
        full = f == K
        kinds[j] = np.where(full, L.KSA_SUMMARY, L.KSA_TEXT)
        f = np.where(full, 0, f + 1)
    return kinds


def _host_image(t: torch.Tensor) -> np.ndarray:
    """[Hkv, S, d] device slice -> contiguous [S, Hkv, d] fp64 on the host."""
    return np.ascontiguousarray(to_f64(t.transpose(0, 1)))


@pytest.mark.parametrize("B,context,watch", POINTS, ids=[f"b{p[0]}_ctx{p[1]}" for p in POINTS])
def test_decode_sweep_schedule_against_cache_model(B, context, watch):
    m0 = context // K
    p = L.make_params(K, W, HQ, HKV, D, 0.0, THETA)
    cache = DecodeCache(p, B, cap=m0 + 2 * (TEXT_STEPS // K))
    fill_normal_(cache.k, 1000 + B)
    fill_normal_(cache.v, 2000 + B)
    fills = uniform_ints(B, 0, K - 1, seed=7).numpy()
    state0 = torch.zeros(B, 4, dtype=torch.int32)
    state0[:, 0] = torch.as_tensor(m0 * K + fills, dtype=torch.int32)
    state0[:, 1] = m0
    cache.state.copy_(state0)
    kinds = _schedule(fills, m0)
    kinds_d = torch.as_tensor(kinds, device="cuda")
    max_text = (m0 + 2 * (TEXT_STEPS // K) + 1) * K
    ws = cache.workspace(max_text)
    gen = torch.Generator(device="cuda").manual_seed(7)
    # The watched sequences' images: the summary region is append-only, so
    # after the first copy only the scratch, open-chunk and ring slots and
    # the newly appended summary slots are read back.
    head = 1 + K + W * K
    imgs = {b: (_host_image(cache.k[b]), _host_image(cache.v[b])) for b in watch}
    rows = RowSet(f"decode sweep b{B} ctx{context}")
    n_summary = 0
    for j in range(kinds.shape[0]):
        kn = torch.randn(B, HKV, D, generator=gen, device="cuda").to(torch.bfloat16)
        vn = torch.randn(B, HKV, D, generator=gen, device="cuda").to(torch.bfloat16)
        q = torch.randn(B, HQ, D, generator=gen, device="cuda").to(torch.bfloat16)
        cache.append(kinds_d[j], kn, vn)
        o, lse = cache.decode(kinds_d[j], q, max_text, ws)
        torch.cuda.synchronize()
        st = cache.state.cpu().numpy()
        assert np.all(st[:, 3] == 0), f"step {j}: state errors {st[:, 3]}"
        og, lg = to_f64(o), to_f64(lse)
        for b in watch:
            Kimg, Vimg = imgs[b]
            m_now = int(st[b, 1])
            for img, src in ((Kimg, cache.k[b]), (Vimg, cache.v[b])):
                img[:head] = _host_image(src[:, :head])
                img[head + m0:head + m_now] = _host_image(src[:, head + m0:head + m_now])
            # the oracle rotates the bf16 input query itself, in fp64, at the
            # position of the step's token (a summary: its chunk's last token)
            qr = oracle.rope(to_f64(q[b])[None], np.array([st[b, 0] - 1]), THETA)[0]
            kd = oracle.TEXT if kinds[j, b] == L.KSA_TEXT else oracle.SUMMARY
            want_o, want_l = oracle.decode_image(K, W, cache.cap, int(st[b, 0]), m_now, kd, Kimg, Vimg, qr)
            rows.add(og[b], want_o, f"step {j} seq {b} kind {kd}")
            assert_close(lg[b], want_l, f"step {j} seq {b} lse", max_abs=LSE_ABS, rel_frob=None)
        n_summary += int((kinds[j] == L.KSA_SUMMARY).sum())
    rows.check()
    st = cache.state.cpu().numpy()
    # every sequence made 64 text and 8 summary steps: the ring wrapped once
    np.testing.assert_array_equal(st[:, 0], m0 * K + fills + TEXT_STEPS)
    np.testing.assert_array_equal(st[:, 1], m0 + TEXT_STEPS // K)
    assert n_summary == B * (TEXT_STEPS // K)
