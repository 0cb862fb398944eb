"""ksa_decode_noalloc: the decode step for callers that cannot allocate
device memory (a host program that owns all of the GPU's memory, or a custom
op handed only its inputs and outputs).  It must give the same results as
ksa_decode with a caller-provided workspace, call after call, although its
scratch is one fixed array the library keeps for the life of the process.

This file is collected last on purpose, so that a stop-at-first-failure run
has already run every other test if this one fails."""
import numpy as np
import pytest
import torch

from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.api import DecodeCache
from kv_cache_compression_ksa_b200.inputs import fill_normal_, uniform_ints
from ksa_testutil import LSE_ABS, MAX_ABS, assert_close, to_f64

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


def test_noalloc_decode_matches_workspace_decode_twice():
    B, m = 16, 300
    p, cache = _cache(B, m)
    gen = torch.Generator(device="cuda").manual_seed(41)
    kind = torch.zeros(B, dtype=torch.int8, device="cuda")
    kn = torch.randn(B, p.num_kv_heads, p.head_dim, generator=gen, device="cuda").to(torch.bfloat16)
    cache.append(kind, kn, kn)
    max_text = m * p.k + p.k
    assert L.ksa_decode_workspace_size(p, B, max_text) <= SCRATCH_LIMIT
    ref_o, ref_l = [], []
    got_o, got_l = [], []
    for call in range(2):
        q = torch.randn(B, p.num_q_heads, p.head_dim, generator=gen, device="cuda").to(torch.bfloat16)
        o1, l1 = cache.decode(kind, q, max_text)            # caller-provided workspace
        o2 = torch.full_like(o1, float("nan"))
        l2 = torch.full_like(l1, float("nan"))
        L.ksa_decode_noalloc(p, cache.desc, kind, q, o2, l2, max_text)
        torch.cuda.synchronize()
        ref_o.append(to_f64(o1)); ref_l.append(to_f64(l1))
        got_o.append(to_f64(o2)); got_l.append(to_f64(l2))
    for call in range(2):
        assert_close(got_o[call], ref_o[call], f"noalloc call {call} O", max_abs=MAX_ABS, rel_frob=None)
        assert_close(got_l[call], ref_l[call], f"noalloc call {call} LSE", max_abs=LSE_ABS, rel_frob=None)
    # the two calls used different queries: the second result is not a stale copy
    assert not np.array_equal(got_o[0], got_o[1])
    assert (cache.state[:, 3] == 0).all()


def test_noalloc_decode_rejects_problems_beyond_its_scratch():
    """A batch whose split-K partials exceed the fixed scratch is refused with
    KSA_ERR_CAPACITY before anything is launched."""
    B, m = 2048, 4
    p = L.make_params(8, 8, 32, 8, 128, 0.0, 1e6)
    max_text = 1 << 20
    assert L.ksa_decode_workspace_size(p, B, max_text) > SCRATCH_LIMIT
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
