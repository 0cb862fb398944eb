"""The C-ABI library loads, exports every symbol include/ksa.h declares, and
rejects bad arguments on the host before launching anything (no GPU needed:
these calls return before their first CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ksa.h")


@pytest.fixture(scope="module")
def lib():
    from kv_cache_compression_ksa_b200 import build, _lib
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*KSA_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*(ksa_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("ksa_interleave_rope", "ksa_prefill_fwd", "ksa_cache_append", "ksa_decode"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), f"libksa.so does not export {n}"


def test_host_side_validation(lib):
    from kv_cache_compression_ksa_b200 import _lib as L
    p = L.make_params(8, 8, 32, 8, 128)
    # sizes
    assert L.ksa_cache_slots(p, 16384) == 1 + 8 + 64 + 16384
    assert L.ksa_aug_rows(p, [32768]) == 36864
    assert L.ksa_aug_rows(p, [131072, 65536, 16384, 4000]) == 244116
    assert L.ksa_aug_rows(p, [4003]) == 501 * 9
    assert L.ksa_prefill_workspace_size(p, 4, 1000) >= 16
    # bad parameters: returned before any launch
    nul = ctypes.c_void_p(0)
    bad = L.make_params(0, 8, 32, 8, 128)
    rc = lib.ksa_prefill_fwd(ctypes.byref(bad), 1, 8, 8, 9, nul, nul, nul, nul, nul, 8, 64, nul, nul)
    assert rc == L.KSA_ERR_INVALID
    odd = L.make_params(8, 8, 32, 8, 96)
    rc = lib.ksa_prefill_fwd(ctypes.byref(odd), 1, 8, 8, 9, nul, nul, nul, nul, nul, 8, 64, nul, nul)
    assert rc == L.KSA_ERR_UNSUPPORTED
    gqa = L.make_params(8, 8, 30, 8, 128)  # 30 % 8 != 0
    rc = lib.ksa_prefill_fwd(ctypes.byref(gqa), 1, 8, 8, 9, nul, nul, nul, nul, nul, 8, 64, nul, nul)
    assert rc == L.KSA_ERR_INVALID
    # null cu_seqlens
    rc = lib.ksa_prefill_fwd(ctypes.byref(p), 1, nul, 8, 9, nul, nul, nul, nul, nul, 16, 4096, nul, nul)
    assert rc == L.KSA_ERR_INVALID
    # aug_rows not a multiple of k+1
    rc = lib.ksa_prefill_fwd(ctypes.byref(p), 1, 16, 8, 10, 16, 16, 16, 16, nul, 16, 4096, nul, nul)
    assert rc == L.KSA_ERR_INVALID
    # workspace too small
    rc = lib.ksa_prefill_fwd(ctypes.byref(p), 1, 16, 8, 9, 16, 16, 16, 16, nul, 16, 8, nul, nul)
    assert rc == L.KSA_ERR_WORKSPACE
    # prefill: k > 128 (a chunk's slots exceed a query tile) and 3 q heads per
    # kv head (no summary-row kernel) are unsupported
    big = L.make_params(129, 1, 8, 2, 128)
    rc = lib.ksa_prefill_fwd(ctypes.byref(big), 1, 16, 129, 130, 16, 16, 16, 16, nul, 16, 4096, nul, nul)
    assert rc == L.KSA_ERR_UNSUPPORTED
    g3 = L.make_params(8, 1, 6, 2, 128)
    rc = lib.ksa_prefill_fwd(ctypes.byref(g3), 1, 16, 8, 9, 16, 16, 16, 16, nul, 16, 4096, nul, nul)
    assert rc == L.KSA_ERR_UNSUPPORTED
    # decode: null cache pointers
    cache = L.ksa_cache(None, None, None, 4, 10)
    rc = lib.ksa_decode(ctypes.byref(p), ctypes.byref(cache), 16, 16, 16, nul, 100, 16, 1 << 20, nul)
    assert rc == L.KSA_ERR_INVALID
    rc = lib.ksa_cache_append(ctypes.byref(p), ctypes.byref(cache), 16, 16, 16, nul)
    assert rc == L.KSA_ERR_INVALID
    assert lib.ksa_get_device_error(nul, nul) == L.KSA_ERR_INVALID
    assert L.status_string(L.KSA_ERR_STATE) == "decode cache order violated"


def test_binding_refuses_host_tensors(lib):
    import torch
    from kv_cache_compression_ksa_b200 import _lib as L
    with pytest.raises(ValueError):
        L._ptr(torch.zeros(4))


def test_binding_checks_element_types(lib):
    """Each tensor argument must have the element type include/ksa.h
    documents (bf16 data, fp32 LSE, int32 offsets / state / error words,
    int8 kinds).  The check runs before the device check, so a wrong type
    is named even on a host without a GPU; an int stands for a raw device
    address and passes through, so the arguments before the one under test
    are given as ints."""
    import torch
    from kv_cache_compression_ksa_b200 import _lib as L
    p = L.make_params(8, 2, 8, 2, 64)
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    cu = torch.tensor([0, 16], dtype=torch.int32)
    ws = torch.zeros(64, dtype=torch.uint8)
    A = 256   # a stand-in device address
    # prefill: int64 offsets are refused by the call; fp16 data and bf16 LSE
    # by the marshalling every call uses
    with pytest.raises(ValueError, match="int32"):
        L.ksa_prefill_fwd(p, cu.long(), 16, 18, A, A, A, A, None, ws)
    with pytest.raises(ValueError, match="bfloat16"):
        L._ptr(bf(18, 8, 64).half(), L.BF16)
    with pytest.raises(ValueError, match="float32"):
        L._ptr(bf(18, 8), L.F32)
    # the right type on the host gets as far as the device check
    with pytest.raises(ValueError, match="CUDA device"):
        L._ptr(torch.zeros(18, 8), L.F32)
    # decode cache: int64 state; int32 / uint8 kinds
    with pytest.raises(ValueError, match="int32"):
        L.make_cache(A, A, torch.zeros(1, 4, dtype=torch.int64), 4)
    cache = L.ksa_cache(0, 0, 0, 1, 4)
    with pytest.raises(ValueError, match="int8"):
        L.ksa_decode(p, cache, torch.zeros(1, dtype=torch.int32), A, A, None, 16, ws)
    with pytest.raises(ValueError, match="int8"):
        L.ksa_cache_append(p, cache, torch.zeros(1, dtype=torch.uint8), A, A)
    # an error word is int32, or the byte workspace that holds the default one
    with pytest.raises(ValueError, match="int32"):
        L.ksa_get_device_error(torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA device"):
        L.ksa_get_device_error(torch.zeros(16, dtype=torch.uint8))
    # MLA: fp32 latent rows
    pm = L.make_mla_params(8, 2, 16)
    mc = L.ksa_mla_cache(0, 0, 1, 4)
    with pytest.raises(ValueError, match="bfloat16"):
        L.ksa_mla_cache_append(pm, mc, A, torch.zeros(1, 576))


def test_window_bound(lib):
    """The kernels index the window ((w + 1) k text tokens) in 32-bit
    arithmetic, so a larger window is refused before any launch instead of
    wrapping; the largest allowed one is accepted."""
    from kv_cache_compression_ksa_b200 import _lib as L
    nul = ctypes.c_void_p(0)
    edge = L.make_params(8, (1 << 27) - 1, 32, 8, 128)       # (w + 1) k = 2^30
    over = L.make_params(8, 1 << 27, 32, 8, 128)
    full = L.make_params(8, 2 ** 31 - 1, 32, 8, 128)        # "every chunk"
    assert L.ksa_decode_workspace_size(edge, 4, 1000) > 0
    assert L.ksa_decode_workspace_size(over, 4, 1000) == 0
    assert L.ksa_prefill_bwd_workspace_size(full, 1, 9) == 0
    for p in (over, full):
        rc = lib.ksa_prefill_fwd(ctypes.byref(p), 1, 8, 8, 9, nul, nul, nul, nul, nul, 8, 64, nul, nul)
        assert rc == L.KSA_ERR_UNSUPPORTED
        cache = L.ksa_cache(16, 16, 16, 1, 4)
        rc = lib.ksa_decode(ctypes.byref(p), ctypes.byref(cache), 16, 16, 16, nul, 100, 16, 1 << 20, nul)
        assert rc == L.KSA_ERR_UNSUPPORTED
    pm = L.make_mla_params(8, 1 << 27, 16)
    assert L.ksa_mla_decode_workspace_size(pm, 4, 1000) == 0
    assert L.ksa_mla_decode_workspace_size(L.make_mla_params(8, (1 << 27) - 1, 16), 4, 1000) > 0


def test_noalloc_decode_checks_arguments_like_decode(lib):
    """The no-workspace decode runs the same argument checks as ksa_decode
    and returns the same status for the same bad call (a window beyond the
    32-bit bound, bad parameters, a missing query, an empty batch), all
    before any launch."""
    from kv_cache_compression_ksa_b200 import _lib as L
    nul = ctypes.c_void_p(0)
    good = L.make_params(8, 8, 32, 8, 128)
    cases = [
        (L.make_params(8, 1 << 27, 32, 8, 128), L.ksa_cache(16, 16, 16, 1, 4), 16, L.KSA_ERR_UNSUPPORTED),
        (L.make_params(0, 8, 32, 8, 128), L.ksa_cache(16, 16, 16, 1, 4), 16, L.KSA_ERR_INVALID),
        (L.make_params(8, 8, 32, 8, 96), L.ksa_cache(16, 16, 16, 1, 4), 16, L.KSA_ERR_UNSUPPORTED),
        (good, L.ksa_cache(16, 16, 16, 1, 4), 0, L.KSA_ERR_INVALID),          # no query
        (good, L.ksa_cache(16, 16, 16, -1, 4), 16, L.KSA_ERR_INVALID),        # negative batch
        (good, L.ksa_cache(0, 0, 0, 0, 4), 0, L.KSA_OK),                      # empty batch: nothing to do
    ]
    for p, cache, q, want in cases:
        rc_ws = lib.ksa_decode(ctypes.byref(p), ctypes.byref(cache), 16, q, 16, nul, 100, 16, 1 << 20, nul)
        rc_na = lib.ksa_decode_noalloc(ctypes.byref(p), ctypes.byref(cache), 16, q, 16, nul, 100, nul)
        assert rc_ws == want and rc_na == want, (p.k, p.w, p.head_dim, cache.batch, rc_ws, rc_na)


def test_noalloc_decode_refuses_a_batch_whose_split_does_not_fit(lib):
    """One split of the partials takes 4 B x batch x Hq x (d + 2); above the
    fixed 4 MiB array (253 sequences x 32 q heads at d 128: 4,209,920 B)
    the no-workspace call refuses with KSA_ERR_CAPACITY, and ksa_decode
    with a workspace too small for it with KSA_ERR_WORKSPACE, both before
    any launch or device access."""
    from kv_cache_compression_ksa_b200 import _lib as L
    nul = ctypes.c_void_p(0)
    p = L.make_params(8, 8, 32, 8, 128)
    cache = L.ksa_cache(16, 16, 16, 253, 4)
    assert 4 * 253 * 32 * (128 + 2) > 4 << 20
    assert lib.ksa_decode_noalloc(ctypes.byref(p), ctypes.byref(cache), 16, 16, 16, nul, 100, nul) == \
        L.KSA_ERR_CAPACITY
    assert lib.ksa_decode(ctypes.byref(p), ctypes.byref(cache), 16, 16, 16, nul, 100, 16, 1 << 20, nul) == \
        L.KSA_ERR_WORKSPACE


def test_selftest_wait_timeout_arguments(lib):
    """The timeout self-check launches one CTA whose waits are bounded by the
    given limits; limits outside (0, the pipelines' own limit] and a missing
    error word are refused before the launch."""
    from kv_cache_compression_ksa_b200 import _lib as L
    nul = ctypes.c_void_p(0)
    word = ctypes.c_void_p(1 << 20)
    assert lib.ksa_selftest_wait_timeout(16, 16, nul, nul) == L.KSA_ERR_INVALID
    assert lib.ksa_selftest_wait_timeout(0, 16, word, nul) == L.KSA_ERR_INVALID
    assert lib.ksa_selftest_wait_timeout(16, 0, word, nul) == L.KSA_ERR_INVALID
    assert lib.ksa_selftest_wait_timeout((1 << 22) + 1, 16, word, nul) == L.KSA_ERR_INVALID
    assert lib.ksa_selftest_wait_timeout(16, (1 << 17) + 1, word, nul) == L.KSA_ERR_INVALID
    assert lib.ksa_selftest_wait_timeout(16, 16, ctypes.c_void_p((1 << 20) + 2), nul) == L.KSA_ERR_INVALID
