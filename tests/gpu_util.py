"""Helpers for the GPU parity tests: move seeded NumPy inputs to the device,
run the library, compare with the oracle under the tolerance rule
max|got - ref| <= tau * max|ref| (tau = 1e-5 for fp32 inputs, 2e-2 for bf16
inputs with fp32 state)."""
import numpy as np
import torch

import oracle

TAU = {"f32": 1e-5, "bf16": 2e-2}


def to_device(d, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32

    def t(a, dt=torch.float32):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dt)

    return dict(X=t(d["X"], tdt), log_a=t(d["log_a"]), B=t(d["B"], tdt), C=t(d["C"], tdt), D=t(d["D"]),
                init_states=t(d["init_states"]),
                seq_idx=None if d["seq_idx"] is None else torch.from_numpy(d["seq_idx"]).to("cuda"),
                nseq=d["nseq"])


def run_gpu(d, dtype, chunk, path="auto"):
    import mamba_ssd_layer_chunked_b200 as ssd
    g = to_device(d, dtype)
    Y, final = ssd.ssd_fwd(g["X"], g["log_a"], g["B"], g["C"], chunk, D=g["D"], init_states=g["init_states"],
                           seq_idx=g["seq_idx"], nseq=g["nseq"] if g["seq_idx"] is not None else None,
                           path=path)
    torch.cuda.synchronize()
    ssd.check_device_error()  # no bounded wait of any kernel gave up
    return Y.float().cpu().numpy().astype(np.float64), final.cpu().numpy().astype(np.float64)


def run_oracle(d):
    return oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"], d["seq_idx"],
                                nseq=d["nseq"])


def rel_err(got, ref):
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return err, scale


def assert_close(got, ref, tau, what, atol=0.0):
    """max|got - ref| <= tau * max|ref| + atol (atol only for quantities that
    fp32 cannot hold, such as decays below its smallest normal number)."""
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err, scale = rel_err(got, ref)
    assert err <= tau * scale + atol, f"{what}: max|d| = {err:.3e} > {tau:g} * max|ref| + {atol:g} = {tau * scale + atol:.3e}"
    return err / scale if scale else 0.0
