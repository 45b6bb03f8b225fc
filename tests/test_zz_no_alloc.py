"""ssd_fwd_noalloc: the forward pass for callers that cannot allocate device
memory (their device memory is planned ahead, or an allocation's implicit
synchronisation is not acceptable). It must give the same result as ssd_fwd,
call after call, while its scratch lives in a fixed array inside the library.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import TAU, assert_close, to_device
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


@pytest.mark.gpu
def test_noalloc_matches_ssd_fwd_on_two_calls_in_a_row():
    ssd, f = _noalloc()
    d = make_custom(2, 1024, 4, 64, 128, dtype="bf16", seed=77, has_D="normal", has_init=True,
                    lengths=[[300, 724], [1024]], nseq=2)
    g = to_device(d, "bf16")
    X, B = g["X"], g["B"]
    Yref, Fref = ssd.ssd_fwd(X, g["log_a"], B, g["C"], 256, D=g["D"], init_states=g["init_states"],
                             seq_idx=g["seq_idx"], nseq=2)
    torch.cuda.synchronize()
    Yref = Yref.float().cpu().numpy().astype(np.float64)
    Fref = Fref.cpu().numpy().astype(np.float64)
    p = ssd.problem_from(X, B, 256, 2)
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        Y = torch.full_like(X, float("nan"))
        F = torch.full((2, 2, 4, 128, 64), float("nan"), dtype=torch.float32, device="cuda")
        st = f(ctypes.byref(p), vp(X), vp(g["log_a"]), vp(B), vp(g["C"]), vp(g["D"]), vp(g["init_states"]),
               vp(g["seq_idx"]), vp(Y), vp(F), stream)
        assert st == SSD_OK, f"call {call}: {ssd.status_string(st)}"
        torch.cuda.synchronize()
        assert_close(Y.float().cpu().numpy().astype(np.float64), Yref, TAU["bf16"], f"Y (call {call})")
        assert_close(F.cpu().numpy().astype(np.float64), Fref, TAU["bf16"], f"final_states (call {call})")
