"""The bounded-wait error path of the tensor-core pipelines, run on the GPU
without any fault: ksa_selftest_wait_timeout waits, with the pipelines' own
wait routines and small limits, on mbarriers that nothing completes.  The
call must return on its own, report KSA_ERR_TIMEOUT through the error word,
leave the context usable, and free the SM's tensor memory: a prefill run
right after it (its CTAs allocate all 512 TMEM columns of their SM) still
matches the oracle."""
import time

import pytest
import torch

from kv_cache_compression_ksa_b200 import _lib as L
from test_gpu_prefill import check_against_oracle, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_waits_time_out_and_release_tmem():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    L.ksa_selftest_wait_timeout(1 << 12, 1 << 4, err)       # at most 4096 polls and 16 sleeps of 20 us
    assert L.ksa_get_device_error(err) == L.KSA_ERR_TIMEOUT
    assert time.monotonic() - t0 < 10.0
    assert L.ksa_get_device_error(err) == L.KSA_OK          # read and cleared
    # the context still works
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2
    # twice in a row, then the full tensor-core prefill on the same device
    L.ksa_selftest_wait_timeout(1 << 12, 1 << 4, err)
    assert L.ksa_get_device_error(err) == L.KSA_ERR_TIMEOUT
    x, out = run_gpu([300, 77], 8, 2, 8, 2, 128, 1.0, 31)
    check_against_oracle(x, out, 8, 2, tag="prefill after the timeout self-check")
