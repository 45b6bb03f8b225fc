"""Single-step decoding (ssd_decode_step): the recurrence one token at a time
with an fp32 state cache. Fed a whole sequence token by token from the
initial state, it must give the oracle's outputs and final state; the host
checks of the entry point run without a GPU."""
import ctypes

import numpy as np
import pytest

import mamba_ssd_layer_chunked_b200 as ssd
from tests.gpu_util import TAU, assert_close, run_oracle
from workloads import make_custom

OK, INVALID, UNSUPPORTED = 0, 1, 2
FAKE = 0x10000


def _prob(**kw):
    base = dict(batch=2, seqlen=64, nheads=4, headdim=64, dstate=128, ngroups=1, chunk=64, nseq=1,
                dtype=ssd.ssd.SSD_DTYPE_BF16, path=0)
    base.update(kw)
    return ssd.Problem(**base)


def _call(p, x=FAKE, la=FAKE, B=FAKE, C=FAKE, D=None, st=FAKE, y=FAKE):
    return ssd.lib().ssd_decode_step(ctypes.byref(p), x, la, B, C, D, st, y, None)


@pytest.mark.parametrize("arg", ["x", "la", "B", "C", "st", "y"])
def test_null_pointer_rejected(arg):
    assert _call(_prob(), **{arg: None}) == INVALID


def test_bad_problem_rejected():
    assert ssd.lib().ssd_decode_step(None, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None) == INVALID
    assert _call(_prob(ngroups=3)) == INVALID
    assert _call(_prob(dtype=7)) == INVALID
    assert _call(_prob(headdim=18)) == UNSUPPORTED
    assert _call(_prob(headdim=2048)) == UNSUPPORTED


@pytest.mark.parametrize("arg,off", [("st", 8), ("x", 4), ("y", 4), ("la", 2), ("D", 2)])
def test_misaligned_pointer_rejected(arg, off):
    assert _call(_prob(), **{arg: FAKE + off}) == INVALID


DECODE_CASES = {
    # name: (batch, T, H, P, N, G, dtype, D, init)
    "f32_small": (2, 40, 3, 16, 16, 1, "f32", "ones", True),
    "f32_P256_N48": (1, 12, 2, 256, 48, 1, "f32", "normal", False),
    "bf16_N128_groups2": (2, 24, 4, 64, 128, 2, "bf16", "normal", True),
    "bf16_N64": (3, 16, 6, 64, 64, 1, "bf16", "none", True),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(DECODE_CASES))
def test_decode_steps_match_the_recurrence(name):
    import torch
    b, T, H, P, N, G, dtype, D, init = DECODE_CASES[name]
    d = make_custom(b, T, H, P, N, ngroups=G, dtype=dtype, seed=500 + T, has_D=D, has_init=init)
    Yr, Fr = run_oracle(d)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt)
    X, la, B, C = dev(d["X"], tdt), dev(d["log_a"]), dev(d["B"], tdt), dev(d["C"], tdt)
    Dt = None if d["D"] is None else dev(d["D"])
    state = (dev(d["init_states"][:, 0]).contiguous() if d["init_states"] is not None
             else torch.zeros(b, H, N, P, dtype=torch.float32, device="cuda"))
    ys = []
    for t in range(T):
        ys.append(ssd.decode_step(X[:, t].contiguous(), la[:, t].contiguous(), B[:, t].contiguous(),
                                  C[:, t].contiguous(), state, D=Dt))
    torch.cuda.synchronize()
    Y = torch.stack(ys, dim=1).float().cpu().numpy().astype(np.float64)
    tau = TAU[dtype]
    assert_close(Y, Yr, tau, "decode y")
    assert_close(state.cpu().numpy().astype(np.float64), Fr[:, 0], tau, "decode final state")


@pytest.mark.gpu
def test_decode_continues_a_prefill():
    """ssd_fwd over a prefix, then decode steps from its final states: the
    outputs equal those of one ssd_fwd over the whole sequence (oracle)."""
    import torch
    b, T, H, P, N = 2, 256 + 8, 4, 64, 128
    d = make_custom(b, T, H, P, N, dtype="bf16", seed=77, has_D="normal", has_init=True)
    Yr, Fr = run_oracle(d)
    dev = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt)
    X, la, B, C = dev(d["X"], torch.bfloat16), dev(d["log_a"]), dev(d["B"], torch.bfloat16), dev(d["C"], torch.bfloat16)
    Dt, init = dev(d["D"]), dev(d["init_states"])
    Y0, F0 = ssd.ssd_fwd(X[:, :256].contiguous(), la[:, :256].contiguous(), B[:, :256].contiguous(),
                         C[:, :256].contiguous(), 128, D=Dt, init_states=init)
    state = F0[:, 0].contiguous()
    ys = [ssd.decode_step(X[:, t].contiguous(), la[:, t].contiguous(), B[:, t].contiguous(), C[:, t].contiguous(),
                          state, D=Dt) for t in range(256, T)]
    torch.cuda.synchronize()
    tau = TAU["bf16"]
    assert_close(Y0.float().cpu().numpy().astype(np.float64), Yr[:, :256], tau, "prefill y")
    assert_close(torch.stack(ys, 1).float().cpu().numpy().astype(np.float64), Yr[:, 256:], tau, "decode y")
    assert_close(state.cpu().numpy().astype(np.float64), Fr[:, 0], tau, "final state")
