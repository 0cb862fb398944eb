"""GPU parity of the KSA decode over an MLA latent cache (Kwai Summary
Attention Technical Report section 3.2, Eq. (6); MLA per section 3.1; slot
map of section 2.3.1, Figure 4): ksa_mla_decode against the oracle's absorbed
decode on seeded cache images, and ksa_mla_cache_append against the oracle's
cache model fed the same tokens."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import MlaCache
from kv_cache_compression_ksa_b200.inputs import fill_normal_, uniform_ints
from ksa_testutil import LSE_ABS, RowSet, assert_close, to_f64

pytestmark = pytest.mark.gpu
THETA = 1e6
DC, DR = 512, 64


def _image_case(B, H, k, w, ms, fills, kinds, seed):
    """A latent cache filled straight from N(0,1) with state {m k + f, m}."""
    p = L.make_mla_params(k, w, H, DC, DR, 0.0, THETA)
    cap = max(ms) + 2
    cache = MlaCache(p, B, cap)
    fill_normal_(cache.latent, seed)
    st = torch.zeros(B, 4, dtype=torch.int32)
    st[:, 0] = torch.as_tensor([m * k + f for m, f in zip(ms, fills)], dtype=torch.int32)
    st[:, 1] = torch.as_tensor(ms, dtype=torch.int32)
    cache.state.copy_(st.cuda())
    gen = torch.Generator(device="cuda").manual_seed(seed + 1)
    q = torch.randn(B, H, DC + DR, generator=gen, device="cuda").to(torch.bfloat16)
    kind = torch.as_tensor(kinds, dtype=torch.int8, device="cuda")
    return p, cap, cache, q, kind


CASES = [
    # B, H, k, w, summaries per sequence, fills (f after the step's append), kinds
    (3, 16, 4, 2, [0, 1, 9], [2, 4, 3], [0, 0, 0]),                 # m < w, m = w - 1, m > w
    (4, 32, 8, 8, [100, 7, 40, 3], [1, 8, 0, 5], [0, 0, 1, 0]),     # a SUMMARY step (f = 0)
    (2, 64, 8, 0, [50, 5], [3, 1], [0, 0]),                         # w = 0
    (3, 128, 8, 8, [2000, 513, 64], [7, 1, 0], [0, 0, 1]),          # Table 1's 128 heads
    (2, 48, 16, 3, [70, 2], [16, 9], [0, 2]),                       # 48 heads (padded group), SKIP
    (2, 256, 8, 8, [300, 1200], [3, 8], [0, 0]),                    # two groups of 128 heads
    (4, 128, 4, 1, [5000, 1, 0, 700], [2, 4, 1, 0], [2, 0, 0, 1]),  # SKIP first, m < w, m = 0, SUMMARY
    (2, 128, 4, 2, [1, 0], [4, 2], [0, 0]),                         # a 16-slot cache: one partial block
]


@pytest.mark.parametrize("B,H,k,w,ms,fills,kinds", CASES)
def test_mla_decode_matches_oracle(B, H, k, w, ms, fills, kinds):
    p, cap, cache, q, kind = _image_case(B, H, k, w, ms, fills, kinds, seed=11 + H)
    max_text = max(m * k + f for m, f in zip(ms, fills))
    o = torch.full((B, H, DC), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H), 7.0, dtype=torch.float32, device="cuda")
    ws = cache.workspace(max_text)
    L.ksa_mla_decode(p, cache.desc, kind, q, o, lse, max_text, ws)
    torch.cuda.synchronize()
    assert (cache.state[:, 3] == 0).all()
    img = to_f64(cache.latent)
    og, lg = to_f64(o), to_f64(lse)
    scale = 1.0 / np.sqrt(DC + DR)
    for b in range(B):
        n = ms[b] * k + fills[b]
        if kinds[b] == L.KSA_SKIP:
            assert (og[b] == 7.0).all() and (lg[b] == 7.0).all()
            continue
        ref_o, ref_l = oracle.mla_decode_image(k, w, cap, n, ms[b], kinds[b], img[b], to_f64(q[b]), scale, THETA,
                                               DC)
        assert_close(og[b], ref_o, f"mla H{H} seq {b}")
        assert_close(lg[b], ref_l, f"mla lse H{H} seq {b}", max_abs=LSE_ABS, rel_frob=None)


def test_mla_append_stream_and_decode():
    """Tokens appended one by one (TEXT, then SUMMARY when a chunk fills)
    land where the oracle's cache model puts them (latent part bit-exact, the
    rotated part within one bf16 rounding), and each decode step matches the
    oracle's decode of its own model."""
    B, H, k, w = 3, 16, 4, 2
    steps = [23, 30, 9]            # text tokens per sequence
    p = L.make_mla_params(k, w, H, DC, DR, 0.0, THETA)
    cap = max(steps) // k + 1
    cache = MlaCache(p, B, cap)
    gen = torch.Generator().manual_seed(5)
    lat_t = [torch.randn(n, DC + DR, generator=gen).to(torch.bfloat16) for n in steps]
    lat_s = [torch.randn(n // k, DC + DR, generator=gen).to(torch.bfloat16) for n in steps]
    qs = [torch.randn(n, H, DC + DR, generator=gen).to(torch.bfloat16) for n in steps]
    qss = [torch.randn(n // k, H, DC + DR, generator=gen).to(torch.bfloat16) for n in steps]
    models = [oracle.Cache(k, w, 1, DC + DR, cap) for _ in range(B)]
    done = [0] * B          # text tokens appended
    pend = [False] * B      # a summary step is next
    scale = 1.0 / np.sqrt(DC + DR)
    max_text = max(steps)
    ws = cache.workspace(max_text)
    rows = RowSet("mla stream decode outputs")
    while any(d < n or pd for d, n, pd in zip(done, steps, pend)):
        kinds, x, qq = [], [], []
        for b in range(B):
            if pend[b]:
                j = done[b] // k - 1
                kinds.append(L.KSA_SUMMARY); x.append(lat_s[b][j]); qq.append(qss[b][j])
            elif done[b] < steps[b]:
                kinds.append(L.KSA_TEXT); x.append(lat_t[b][done[b]]); qq.append(qs[b][done[b]])
            else:
                kinds.append(L.KSA_SKIP); x.append(lat_t[b][0]); qq.append(qs[b][0])
        kind = torch.as_tensor(kinds, dtype=torch.int8, device="cuda")
        cache.append(kind, torch.stack(x).cuda())
        o, lse = cache.decode(kind, torch.stack(qq).cuda(), max_text, ws=ws)
        o, lse = to_f64(o), to_f64(lse)
        for b in range(B):
            if kinds[b] == L.KSA_SKIP:
                continue
            mdl = models[b]
            if kinds[b] == L.KSA_TEXT:
                i = done[b]
                K, V = oracle.mla_kv_rows(to_f64(x[b])[None], [i], THETA, DC)
                assert mdl.append_text(K, V) == 0
                done[b] += 1
                pend[b] = done[b] % k == 0
            else:
                K, V = oracle.mla_kv_rows(to_f64(x[b])[None], [done[b] - 1], THETA, DC)
                assert mdl.append_summary(K, V) == 0
                pend[b] = False
            ref_o, ref_l = oracle.mla_decode_image(k, w, cap, mdl.n_text, mdl.m, kinds[b], mdl.K()[:, 0],
                                                   to_f64(qq[b]), scale, THETA, DC)
            rows.add(o[b], ref_o, f"stream seq {b} step {mdl.n_text}/{mdl.m}")
            assert_close(lse[b], ref_l, "stream lse", max_abs=LSE_ABS, rel_frob=None)
    rows.check()
    assert (cache.state[:, 3] == 0).all()
    img = to_f64(cache.latent)
    for b in range(B):
        n, m = steps[b], steps[b] // k
        f = n - m * k
        slots = [k - r for r in range(f)] + [1 + k + w * k + j for j in range(m)]
        if w > 0:
            for c in range(max(0, m - w), m):
                slots += [k + 1 + (c % w) * k + i for i in range(k)]
        slots = np.asarray(sorted(slots))
        want = models[b].K()[slots, 0]
        np.testing.assert_array_equal(img[b][slots, :DC], want[:, :DC])
        assert np.abs(img[b][slots, DC:] - want[:, DC:]).max() <= 0.02 * max(1.0, np.abs(want[:, DC:]).max())


def test_mla_full_size_sampled():
    """16 sequences x 131072 prior tokens (16384 summaries + a full 64-token
    ring), Table 1's 128 heads: every head of four sequences against the
    oracle."""
    B, H, k, w = 16, 128, 8, 8
    ms = [16384] * B
    fills = list(uniform_ints(B, 1, k, seed=3).numpy())
    p, cap, cache, q, kind = _image_case(B, H, k, w, ms, fills, [L.KSA_TEXT] * B, seed=21)
    o, lse = cache.decode(kind, q, max(ms) * k + k)
    torch.cuda.synchronize()
    assert (cache.state[:, 3] == 0).all()
    og, lg = to_f64(o), to_f64(lse)
    scale = 1.0 / np.sqrt(DC + DR)
    for b in (0, 5, 10, 15):
        img = to_f64(cache.latent[b])
        ref_o, ref_l = oracle.mla_decode_image(k, w, cap, ms[b] * k + fills[b], ms[b], L.KSA_TEXT, img,
                                               to_f64(q[b]), scale, THETA, DC)
        assert_close(og[b], ref_o, f"full-size mla seq {b}")
        assert_close(lg[b], ref_l, f"full-size mla lse seq {b}", max_abs=LSE_ABS, rel_frob=None)


def test_mla_state_errors():
    """A SUMMARY step on a sequence whose chunk is not full, and a summary
    past the capacity, are flagged per sequence; the others are served."""
    B, H, k, w = 2, 16, 4, 2
    p = L.make_mla_params(k, w, H, DC, DR, 0.0, THETA)
    cache = MlaCache(p, B, cap=1)
    x = torch.randn(B, DC + DR, device="cuda").to(torch.bfloat16)
    text = torch.full((B,), L.KSA_TEXT, dtype=torch.int8, device="cuda")
    for _ in range(k):
        cache.append(text, x)
    summ = torch.full((B,), L.KSA_SUMMARY, dtype=torch.int8, device="cuda")
    cache.append(summ, x)                                    # both fine: m = 1 = cap
    cache.append(torch.as_tensor([L.KSA_SUMMARY, L.KSA_TEXT], dtype=torch.int8, device="cuda"), x)
    torch.cuda.synchronize()
    st = cache.state.cpu().numpy()
    assert st[0, 3] == L.KSA_ERR_STATE and tuple(st[1, :2]) == (k + 1, 1) and st[1, 3] == 0
    for _ in range(k - 1):
        cache.append(torch.as_tensor([L.KSA_SKIP, L.KSA_TEXT], dtype=torch.int8, device="cuda"), x)
    cache.append(torch.as_tensor([L.KSA_SKIP, L.KSA_SUMMARY], dtype=torch.int8, device="cuda"), x)
    torch.cuda.synchronize()
    assert cache.state[1, 3].item() == L.KSA_ERR_CAPACITY
