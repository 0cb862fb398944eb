"""ctypes binding of libksa.so.  Argument marshalling only: every step of the
KSA path runs in the library's CUDA kernels.  The functions carry the C names
and take torch tensors (device memory) in place of raw pointers.

There is no fallback: if libksa.so is missing or no CUDA device is present,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libksa.so")

KSA_OK = 0
KSA_ERR_INVALID = -1
KSA_ERR_UNSUPPORTED = -2
KSA_ERR_CAPACITY = -3
KSA_ERR_CUDA = -4
KSA_ERR_TIMEOUT = -5
KSA_ERR_WORKSPACE = -6
KSA_ERR_STATE = -7

KSA_TEXT, KSA_SUMMARY, KSA_SKIP = 0, 1, 2


class ksa_params(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_int32),
        ("w", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("rope_theta", ctypes.c_double),
    ]


class ksa_cache(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("state", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("cap_summaries", ctypes.c_int64),
    ]


class KsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")
        self.status = status


class ksa_mla_params(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_int32),
        ("w", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("kv_lora_rank", ctypes.c_int32),
        ("rope_dim", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("rope_theta", ctypes.c_double),
    ]


class ksa_mla_cache(ctypes.Structure):
    _fields_ = [
        ("latent", ctypes.c_void_p),
        ("state", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("cap_summaries", ctypes.c_int64),
    ]


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

SYMBOLS = {
    # name: (restype, argtypes)
    "ksa_aug_rows": (_I64, [ctypes.POINTER(ksa_params), _I32, ctypes.POINTER(_I32)]),
    "ksa_prefill_workspace_size": (_SZ, [ctypes.POINTER(ksa_params), _I32, _I64]),
    "ksa_interleave_rope": (ctypes.c_int, [ctypes.POINTER(ksa_params), _I32, _P, _I64, _I64, _I64,
                                           _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "ksa_interleave_rope_bwd": (ctypes.c_int, [ctypes.POINTER(ksa_params), _I32, _P, _I64, _I64, _I64,
                                               _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "ksa_prefill_fwd": (ctypes.c_int, [ctypes.POINTER(ksa_params), _I32, _P, _I64, _I64,
                                       _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "ksa_prefill_bwd_workspace_size": (_SZ, [ctypes.POINTER(ksa_params), _I32, _I64]),
    "ksa_prefill_bwd": (ctypes.c_int, [ctypes.POINTER(ksa_params), _I32, _P, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _P, _SZ, _P, _P]),
    "ksa_cache_slots": (_I64, [ctypes.POINTER(ksa_params), _I64]),
    "ksa_cache_append": (ctypes.c_int, [ctypes.POINTER(ksa_params), ctypes.POINTER(ksa_cache), _P, _P, _P, _P]),
    "ksa_cache_from_prefill": (ctypes.c_int, [ctypes.POINTER(ksa_params), ctypes.POINTER(ksa_cache), _P, _I64, _I64,
                                              _P, _P, _P, _SZ, _P, _P]),
    "ksa_prefill_chunk_workspace_size": (_SZ, [ctypes.POINTER(ksa_params), _I32, _I64, _I64]),
    "ksa_prefill_chunk": (ctypes.c_int, [ctypes.POINTER(ksa_params), ctypes.POINTER(ksa_cache), _P, _I64, _P, _I64,
                                         _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "ksa_decode_workspace_size": (_SZ, [ctypes.POINTER(ksa_params), _I32, _I64]),
    "ksa_decode": (ctypes.c_int, [ctypes.POINTER(ksa_params), ctypes.POINTER(ksa_cache), _P, _P, _P, _P,
                                  _I64, _P, _SZ, _P]),
    "ksa_decode_noalloc": (ctypes.c_int, [ctypes.POINTER(ksa_params), ctypes.POINTER(ksa_cache), _P, _P, _P, _P,
                                          _I64, _P]),
    "ksa_mla_cache_slots": (_I64, [ctypes.POINTER(ksa_mla_params), _I64]),
    "ksa_mla_cache_append": (ctypes.c_int, [ctypes.POINTER(ksa_mla_params), ctypes.POINTER(ksa_mla_cache), _P, _P,
                                            _P]),
    "ksa_mla_decode_workspace_size": (_SZ, [ctypes.POINTER(ksa_mla_params), _I32, _I64]),
    "ksa_mla_decode": (ctypes.c_int, [ctypes.POINTER(ksa_mla_params), ctypes.POINTER(ksa_mla_cache), _P, _P, _P, _P,
                                      _I64, _P, _SZ, _P]),
    "ksa_get_device_error": (ctypes.c_int, [_P, _P]),
    "ksa_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_uint32, _P, _P]),
    "ksa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}


def load(path: str = LIB_PATH):
    """Load libksa.so (raises OSError if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"libksa.so not built at {path}: run kv_cache_compression_ksa_b200/build.py")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SYMBOLS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    try:
        return load().ksa_status_string(status).decode()
    except OSError:
        return "library not loaded"


# element types the ABI documents for its tensor arguments (include/ksa.h)
BF16, F32, I32, I8 = torch.bfloat16, torch.float32, torch.int32, torch.int8


def _ptr(t, dtype=None):
    """Device pointer of a contiguous CUDA tensor of the given element type
    (None: any, e.g. a byte workspace).  An int passes through as a raw
    device address."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"tensor must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != KSA_OK:
        raise KsaError(fn, rc)


def make_params(k: int, w: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                scale: float = 0.0, rope_theta: float = 1e6) -> ksa_params:
    return ksa_params(k, w, num_q_heads, num_kv_heads, head_dim, scale, rope_theta)


def ksa_aug_rows(p: ksa_params, seqlens) -> int:
    arr = (ctypes.c_int32 * len(seqlens))(*[int(x) for x in seqlens])
    return int(load().ksa_aug_rows(ctypes.byref(p), len(seqlens), arr))


def ksa_prefill_workspace_size(p: ksa_params, batch: int, total_text: int) -> int:
    return int(load().ksa_prefill_workspace_size(ctypes.byref(p), batch, total_text))


def ksa_interleave_rope(p, cu_seqlens, total_text, total_sum, aug_rows, q_text, k_text, v_text,
                        q_sum, k_sum, v_sum, q_aug, k_aug, v_aug, workspace, dev_err=None, stream=None):
    rc = load().ksa_interleave_rope(
        ctypes.byref(p), cu_seqlens.numel() - 1, _ptr(cu_seqlens, I32), total_text, total_sum, aug_rows,
        _ptr(q_text, BF16), _ptr(k_text, BF16), _ptr(v_text, BF16), _ptr(q_sum, BF16), _ptr(k_sum, BF16),
        _ptr(v_sum, BF16), _ptr(q_aug, BF16), _ptr(k_aug, BF16), _ptr(v_aug, BF16), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_err, I32), _stream(stream))
    _check("ksa_interleave_rope", rc)


def ksa_interleave_rope_bwd(p, cu_seqlens, total_text, total_sum, aug_rows, dq_aug, dk_aug, dv_aug,
                            dq_text, dk_text, dv_text, dq_sum, dk_sum, dv_sum, workspace, dev_err=None, stream=None):
    rc = load().ksa_interleave_rope_bwd(
        ctypes.byref(p), cu_seqlens.numel() - 1, _ptr(cu_seqlens, I32), total_text, total_sum, aug_rows,
        _ptr(dq_aug, BF16), _ptr(dk_aug, BF16), _ptr(dv_aug, BF16), _ptr(dq_text, BF16), _ptr(dk_text, BF16),
        _ptr(dv_text, BF16), _ptr(dq_sum, BF16), _ptr(dk_sum, BF16), _ptr(dv_sum, BF16), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_err, I32), _stream(stream))
    _check("ksa_interleave_rope_bwd", rc)


def ksa_prefill_fwd(p, cu_seqlens, total_text, aug_rows, q_aug, k_aug, v_aug, o_aug, lse, workspace,
                    dev_err=None, stream=None):
    rc = load().ksa_prefill_fwd(
        ctypes.byref(p), cu_seqlens.numel() - 1, _ptr(cu_seqlens, I32), total_text, aug_rows,
        _ptr(q_aug, BF16), _ptr(k_aug, BF16), _ptr(v_aug, BF16), _ptr(o_aug, BF16), _ptr(lse, F32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_err, I32), _stream(stream))
    _check("ksa_prefill_fwd", rc)


def ksa_prefill_bwd_workspace_size(p: ksa_params, batch: int, aug_rows: int) -> int:
    return int(load().ksa_prefill_bwd_workspace_size(ctypes.byref(p), batch, aug_rows))


def ksa_prefill_bwd(p, cu_seqlens, total_text, aug_rows, q_aug, k_aug, v_aug, o_aug, lse, do_aug, dq_aug, dk_aug,
                    dv_aug, workspace, dev_err=None, stream=None):
    rc = load().ksa_prefill_bwd(
        ctypes.byref(p), cu_seqlens.numel() - 1, _ptr(cu_seqlens, I32), total_text, aug_rows, _ptr(q_aug, BF16),
        _ptr(k_aug, BF16), _ptr(v_aug, BF16), _ptr(o_aug, BF16), _ptr(lse, F32), _ptr(do_aug, BF16),
        _ptr(dq_aug, BF16), _ptr(dk_aug, BF16), _ptr(dv_aug, BF16), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_err, I32), _stream(stream))
    _check("ksa_prefill_bwd", rc)


def ksa_cache_slots(p: ksa_params, cap_summaries: int) -> int:
    return int(load().ksa_cache_slots(ctypes.byref(p), cap_summaries))


def make_cache(k, v, state, cap_summaries) -> ksa_cache:
    return ksa_cache(_ptr(k, BF16), _ptr(v, BF16), _ptr(state, I32), state.shape[0], cap_summaries)


def ksa_cache_append(p, cache: ksa_cache, kind, k_new, v_new, stream=None):
    rc = load().ksa_cache_append(ctypes.byref(p), ctypes.byref(cache), _ptr(kind, I8), _ptr(k_new, BF16),
                                 _ptr(v_new, BF16), _stream(stream))
    _check("ksa_cache_append", rc)


def ksa_cache_from_prefill(p, cache: ksa_cache, cu_seqlens, total_text, aug_rows, k_aug, v_aug, workspace,
                           dev_err=None, stream=None):
    rc = load().ksa_cache_from_prefill(ctypes.byref(p), ctypes.byref(cache), _ptr(cu_seqlens, I32), total_text,
                                       aug_rows, _ptr(k_aug, BF16), _ptr(v_aug, BF16), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _ptr(dev_err, I32),
                                       _stream(stream))
    _check("ksa_cache_from_prefill", rc)


def ksa_prefill_chunk_workspace_size(p: ksa_params, batch: int, total_text: int, total_sum: int) -> int:
    return int(load().ksa_prefill_chunk_workspace_size(ctypes.byref(p), batch, total_text, total_sum))


def ksa_prefill_chunk(p, cache: ksa_cache, cu_text, total_text, cu_sum, total_sum, q_text, k_text, v_text, q_sum,
                      k_sum, v_sum, o_text, o_sum, lse_text, lse_sum, workspace, dev_err=None, stream=None):
    rc = load().ksa_prefill_chunk(
        ctypes.byref(p), ctypes.byref(cache), _ptr(cu_text, I32), total_text, _ptr(cu_sum, I32), total_sum,
        _ptr(q_text, BF16), _ptr(k_text, BF16), _ptr(v_text, BF16), _ptr(q_sum, BF16), _ptr(k_sum, BF16),
        _ptr(v_sum, BF16), _ptr(o_text, BF16), _ptr(o_sum, BF16), _ptr(lse_text, F32), _ptr(lse_sum, F32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_err, I32), _stream(stream))
    _check("ksa_prefill_chunk", rc)


def ksa_decode_workspace_size(p: ksa_params, batch: int, max_text: int) -> int:
    return int(load().ksa_decode_workspace_size(ctypes.byref(p), batch, max_text))


def ksa_decode(p, cache: ksa_cache, kind, q, o, lse, max_text, workspace, stream=None):
    rc = load().ksa_decode(ctypes.byref(p), ctypes.byref(cache), _ptr(kind, I8), _ptr(q, BF16), _ptr(o, BF16),
                           _ptr(lse, F32), max_text, _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check("ksa_decode", rc)


def ksa_decode_noalloc(p, cache: ksa_cache, kind, q, o, lse, max_text, stream=None):
    """ksa_decode with the library's own fixed scratch instead of a workspace."""
    rc = load().ksa_decode_noalloc(ctypes.byref(p), ctypes.byref(cache), _ptr(kind, I8), _ptr(q, BF16),
                                   _ptr(o, BF16), _ptr(lse, F32), max_text, _stream(stream))
    _check("ksa_decode_noalloc", rc)


def make_mla_params(k: int, w: int, num_heads: int, kv_lora_rank: int = 512, rope_dim: int = 64,
                    scale: float = 0.0, rope_theta: float = 1e6) -> ksa_mla_params:
    return ksa_mla_params(k, w, num_heads, kv_lora_rank, rope_dim, scale, rope_theta)


def make_mla_cache(latent, state, cap_summaries) -> ksa_mla_cache:
    return ksa_mla_cache(_ptr(latent, BF16), _ptr(state, I32), state.shape[0], cap_summaries)


def ksa_mla_cache_slots(p: ksa_mla_params, cap_summaries: int) -> int:
    return int(load().ksa_mla_cache_slots(ctypes.byref(p), cap_summaries))


def ksa_mla_cache_append(p, cache: ksa_mla_cache, kind, x, stream=None):
    rc = load().ksa_mla_cache_append(ctypes.byref(p), ctypes.byref(cache), _ptr(kind, I8), _ptr(x, BF16),
                                     _stream(stream))
    _check("ksa_mla_cache_append", rc)


def ksa_mla_decode_workspace_size(p: ksa_mla_params, batch: int, max_text: int) -> int:
    return int(load().ksa_mla_decode_workspace_size(ctypes.byref(p), batch, max_text))


def ksa_mla_decode(p, cache: ksa_mla_cache, kind, q, o, lse, max_text, workspace, stream=None):
    rc = load().ksa_mla_decode(ctypes.byref(p), ctypes.byref(cache), _ptr(kind, I8), _ptr(q, BF16),
                               _ptr(o, BF16), _ptr(lse, F32), max_text, _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check("ksa_mla_decode", rc)


def ksa_selftest_wait_timeout(poll_limit: int, sleep_limit: int, dev_err, stream=None):
    """Run the bounded-wait self-check: its waits run out and record
    KSA_ERR_TIMEOUT in dev_err (an int32 device word)."""
    rc = load().ksa_selftest_wait_timeout(poll_limit, sleep_limit, _ptr(dev_err, I32), _stream(stream))
    _check("ksa_selftest_wait_timeout", rc)


def ksa_get_device_error(dev_err, stream=None) -> int:
    """Read and clear a device error word: an int32 word, or a byte
    workspace whose first word the calls used because they were given none."""
    ptr = _ptr(dev_err) if isinstance(dev_err, torch.Tensor) and dev_err.dtype == torch.uint8 else _ptr(dev_err, I32)
    return int(load().ksa_get_device_error(ptr, _stream(stream)))
