"""Kwai Summary Attention (KSA) hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libksa.so`` (hand-written CUDA; C ABI in
``include/ksa.h``).  This package holds the ctypes binding (``_lib``), a
thin tensor-level wrapper (``api``), the build script and the seeded
synthetic-input generators (``inputs``).
"""
from . import _lib  # noqa: F401
from ._lib import (  # noqa: F401
    KSA_OK, KSA_TEXT, KSA_SUMMARY, KSA_SKIP, KsaError, ksa_params, ksa_cache, make_params,
    ksa_aug_rows, ksa_prefill_workspace_size, ksa_interleave_rope, ksa_prefill_fwd,
    ksa_cache_slots, ksa_cache_append, ksa_decode_workspace_size, ksa_decode,
    ksa_get_device_error, make_cache,
)
