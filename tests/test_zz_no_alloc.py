"""ssd_fwd_noalloc: the forward pass for callers that cannot allocate device
memory (their device memory is planned ahead, or an allocation's implicit
synchronisation is not acceptable). Its scratch lives in a fixed array inside
the library instead of a caller workspace; it must give ssd_fwd's result bit
for bit, call after call, whatever an earlier call left in that array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import TAU, assert_close, run_oracle, to_device
from workloads import make_custom

SSD_OK, SSD_ERR_WORKSPACE = 0, 3
FAKE = 0x10000  # aligned fake device address; the host checks reject before any use


def _noalloc():
    import mamba_ssd_layer_chunked_b200 as ssd
    f = ssd.lib().ssd_fwd_noalloc
    f.argtypes = [ctypes.POINTER(ssd.Problem)] + [ctypes.c_void_p] * 10
    f.restype = ctypes.c_int
    return ssd, f


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    ssd, f = _noalloc()
    # the 2.7B-shaped layer in fp32 (the SIMT family) needs ~173 MB of scratch
    # (one state per chunk), more than the 64 MiB array: rejected before any launch
    p = ssd.make_problem(4, 4096, 80, 64, 128, 1, 256, 1, torch.float32)
    assert ssd.workspace_bytes(p) > 64 << 20
    assert f(ctypes.byref(p), *([FAKE] * 4), None, None, None, FAKE, None, None) == SSD_ERR_WORKSPACE


def _call(ssd, f, g, chunk, nseq):
    X, B = g["X"], g["B"]
    b, T, H, P = X.shape
    N = B.shape[3]
    p = ssd.problem_from(X, B, chunk, nseq)
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    Y = torch.full_like(X, float("nan"))
    F = torch.full((b, nseq, H, N, P), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = f(ctypes.byref(p), vp(X), vp(g["log_a"]), vp(B), vp(g["C"]), vp(g["D"]), vp(g["init_states"]),
           vp(g["seq_idx"]), vp(Y), vp(F), stream)
    assert st == SSD_OK, ssd.status_string(st)
    return Y, F


@pytest.mark.gpu
def test_noalloc_matches_ssd_fwd_on_two_calls_in_a_row():
    ssd, f = _noalloc()
    d = make_custom(2, 1024, 4, 64, 128, dtype="bf16", seed=77, has_D="normal", has_init=True,
                    lengths=[[300, 724], [1024]], nseq=2)
    g = to_device(d, "bf16")
    Yref, Fref = ssd.ssd_fwd(g["X"], g["log_a"], g["B"], g["C"], 256, D=g["D"], init_states=g["init_states"],
                             seq_idx=g["seq_idx"], nseq=2)
    # first fill the scratch array with another problem's values: a longer row
    # with other boundaries, so its work ranges and cut states cover (and
    # overrun) the regions the target problem uses
    o = make_custom(2, 1536, 4, 64, 128, dtype="bf16", seed=78, has_D="normal", has_init=True,
                    lengths=[[100, 1436], [700, 836]], nseq=2)
    go = to_device(o, "bf16")
    Yo, Fo = _call(ssd, f, go, 256, 2)
    torch.cuda.synchronize()
    Yor, For = run_oracle(o)
    assert_close(Yo.float().cpu().numpy().astype(np.float64), Yor, TAU["bf16"], "Y (other problem)")
    assert_close(Fo.cpu().numpy().astype(np.float64), For, TAU["bf16"], "final_states (other problem)")
    Yr, Fr = run_oracle(d)
    for call in range(2):
        Y, F = _call(ssd, f, g, 256, 2)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: bit for bit what ssd_fwd gives
        assert torch.equal(Y, Yref), f"Y differs from ssd_fwd (call {call})"
        assert torch.equal(F, Fref), f"final_states differ from ssd_fwd (call {call})"
        assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, TAU["bf16"], f"Y vs oracle (call {call})")
        assert_close(F.cpu().numpy().astype(np.float64), Fr, TAU["bf16"], f"final_states vs oracle (call {call})")
    assert ssd.device_error() == 0
