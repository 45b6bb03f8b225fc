"""The failure report of the kernels' bounded waits (ssd_device_error).

Every wait of the tensor-core kernels on a shared-memory barrier is bounded; a
wait that gives up sets a bit of the library's device error word and lets its
CTA finish, so that the host learns of it instead of the GPU hanging. These
tests make one wait give up on purpose, in a dedicated self-test kernel whose
barrier nothing completes (no production kernel is made to time out), and
check that the report reaches the host once, is cleared by reading it, and
leaves the device usable.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import TAU, assert_close, run_gpu, run_oracle
from workloads import make_custom

INVALID, DEVICE_TIMEOUT = 1, 5


def test_selftest_limit_is_checked_on_the_host():
    import mamba_ssd_layer_chunked_b200 as ssd
    lib = ssd.lib()
    # outside 1 us .. 1 s: rejected before anything is launched (safe without a GPU)
    assert lib.ssd_selftest_wait_timeout(999, None) == INVALID
    assert lib.ssd_selftest_wait_timeout(1_000_000_001, None) == INVALID


@pytest.mark.gpu
def test_wait_timeout_is_reported_once_and_the_device_stays_usable():
    import mamba_ssd_layer_chunked_b200 as ssd
    assert ssd.device_error() == 0, "error word set before the test"
    limit_ns = 2_000_000  # 2 ms
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    ssd.selftest_wait_timeout(limit_ns)
    e1.record(s)
    code = ctypes.c_uint32(0)
    st = ssd.lib().ssd_device_error(ctypes.byref(code), ctypes.c_void_p(s.cuda_stream))
    assert st == DEVICE_TIMEOUT and code.value & 1, (st, code.value)
    # the wait honoured its limit before giving up
    assert e0.elapsed_time(e1) >= 0.9 * limit_ns / 1e6
    # reading cleared the word
    assert ssd.device_error() == 0
    # a forward pass after it runs normally, is correct, and reports nothing
    d = make_custom(2, 700, 4, 64, 128, dtype="bf16", seed=5, has_D="normal", has_init=True,
                    lengths=[[300, 400], [700]], nseq=2)
    Y, F = run_gpu(d, "bf16", 256, "fused")
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU["bf16"], "Y")
    assert_close(F, Fr, TAU["bf16"], "final_states")
    assert np.isfinite(Y).all()
