"""The discretisation step (ssd_discretize): the oracle pinned to closed forms
and to the pages' gated-RNN reduction, then the CUDA kernel against the oracle,
alone and feeding ssd_fwd."""
import ctypes

import numpy as np
import pytest

import oracle
from tests.gpu_util import TAU, assert_close
from workloads import make_custom


# --------------------------------------------------------------------------- #
# Pins of the oracle (CPU)
# --------------------------------------------------------------------------- #

def test_softplus_closed_forms():
    dt = np.array([[[0.0, 50.0, -50.0]]])
    A = np.array([-1.0, -1.0, -1.0])
    x = np.ones((1, 1, 3, 4))
    log_a, X = oracle.discretize(dt, A, x)
    delta = -log_a[0, 0]
    assert delta[0] == pytest.approx(np.log(2.0), rel=1e-15)       # softplus(0) = ln 2
    assert delta[1] == pytest.approx(50.0, rel=1e-15)              # softplus(z) -> z
    assert delta[2] == pytest.approx(np.exp(-50.0), rel=1e-12)     # softplus(z) -> e^z
    assert np.allclose(X[0, 0], delta[:, None])                    # Euler: x scaled by delta
    _, Xb = oracle.discretize(dt, A, x, dt_bias=np.array([1.0, 0.0, 0.0]))
    assert Xb[0, 0, 0, 0] == pytest.approx(np.log1p(np.e), rel=1e-15)  # bias added before softplus


def test_zero_order_hold_limits():
    rng = np.random.default_rng(3)
    dt = rng.normal(-3, 1, (2, 5, 4))
    x = rng.normal(0, 1, (2, 5, 4, 8))
    # A = 0: no decay, and the hold factor tends to delta
    la0, X0 = oracle.discretize(dt, np.zeros(4), x, zoh=True)
    _, Xe = oracle.discretize(dt, np.zeros(4), x, zoh=False)
    assert np.all(la0 == 0.0) and np.allclose(X0, Xe, rtol=1e-15)
    # small delta A: (e^{dA} - 1) / A = delta (1 + dA/2 + ...)
    A = np.full(4, -1e-4)
    la, Xz = oracle.discretize(dt, A, x, zoh=True)
    delta = -la / 1e-4
    assert np.allclose(Xz, (delta * (1 + la / 2))[..., None] * x, rtol=1e-8)


def test_gated_rnn_reduction():
    """N = 1, A = -1, B = C = 1 with the zero-order hold: the selective SSM is
    the gated RNN h_t = (1 - g_t) h_{t-1} + g_t x_t with g_t = sigmoid(z_t)
    (the Mamba page's connection to gated RNNs)."""
    rng = np.random.default_rng(11)
    b, T, H, P = 2, 30, 3, 5
    z = rng.normal(0, 2, (b, T, H))
    x = rng.normal(0, 1, (b, T, H, P))
    log_a, X = oracle.discretize(z, -np.ones(H), x, zoh=True)
    ones = np.ones((b, T, 1, 1))
    Y, _ = oracle.ssd_reference(X, log_a, ones, ones, None, None, None)
    g = 1.0 / (1.0 + np.exp(-z))
    h = np.zeros((b, H, P))
    for t in range(T):
        h = (1 - g[:, t, :, None]) * h + g[:, t, :, None] * x[:, t]
        assert np.allclose(Y[:, t], h, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------- #
# Host checks (CPU) and the kernel against the oracle (GPU)
# --------------------------------------------------------------------------- #

def test_host_checks():
    import mamba_ssd_layer_chunked_b200 as ssd
    lib = ssd.lib()
    FAKE = 0x10000
    p = ssd.Problem(1, 64, 2, 64, 16, 1, 64, 1, ssd.ssd.SSD_DTYPE_BF16, 0)
    call = lambda p, dt=FAKE, bias=None, A=FAKE, x=FAKE, la=FAKE, X=FAKE: lib.ssd_discretize(
        ctypes.byref(p), dt, bias, A, x, 0, la, X, None)
    assert call(p, dt=None) == 1 and call(p, A=None) == 1 and call(p, x=None) == 1
    assert call(p, la=None) == 1 and call(p, X=None) == 1
    assert call(p, dt=FAKE + 2) == 1 and call(p, x=FAKE + 1) == 1
    q = ssd.Problem(1, 64, 2, 18, 16, 1, 64, 1, ssd.ssd.SSD_DTYPE_BF16, 0)
    assert call(q) == 2  # headdim not a multiple of 4
    q = ssd.Problem(1, 64, 2, 20, 16, 1, 64, 1, ssd.ssd.SSD_DTYPE_BF16, 0)
    assert call(q) == 2  # bf16 rows of 40 bytes: not whole 16-byte groups
    assert call(p, x=FAKE + 8) == 1 and call(p, X=FAKE + 8) == 1  # x, X 16-byte aligned
    assert lib.ssd_discretize(None, FAKE, None, FAKE, FAKE, 0, FAKE, FAKE, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("bias", [False, True])
def test_kernel_matches_oracle(dtype, zoh, bias):
    import torch
    import mamba_ssd_layer_chunked_b200 as ssd
    rng = np.random.default_rng(100 + 2 * zoh + bias)
    b, T, H, P = 2, 300, 6, 64
    dt = rng.normal(-3, 2, (b, T, H)).astype(np.float32)
    A = -np.exp(rng.uniform(0, np.log(16), H)).astype(np.float32)
    A[1] = 0.0  # no decay on one head
    db = rng.normal(0, 1, H).astype(np.float32) if bias else None
    x = rng.normal(0, 1, (b, T, H, P)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    xg = torch.from_numpy(x).cuda().to(tdt)
    xr = xg.float().cpu().numpy().astype(np.float64)  # the rounded input both sides read
    la, X = ssd.discretize(torch.from_numpy(dt).cuda(), torch.from_numpy(A).cuda(), xg,
                           dt_bias=None if db is None else torch.from_numpy(db).cuda(), zoh=zoh)
    torch.cuda.synchronize()
    la_r, X_r = oracle.discretize(dt, A, xr, db, zoh=zoh)
    assert_close(la.cpu().numpy().astype(np.float64), la_r, 1e-6, "log a")
    assert_close(X.float().cpu().numpy().astype(np.float64), X_r, 1e-6 if dtype == "f32" else 4e-3, "X")


@pytest.mark.gpu
def test_discretize_then_scan():
    """discretize -> ssd_fwd on the GPU against oracle.discretize ->
    oracle.ssd_reference on the same inputs."""
    import torch
    import mamba_ssd_layer_chunked_b200 as ssd
    b, T, H, P, N = 2, 512, 4, 64, 128
    d = make_custom(b, T, H, P, N, dtype="bf16", seed=9, has_D="normal", has_init=True)
    rng = np.random.default_rng(9)
    dt = rng.normal(-3, 1, (b, T, H)).astype(np.float32)
    A = -np.exp(rng.uniform(0, np.log(16), H)).astype(np.float32)
    g = lambda a, t=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(t)
    la, X = ssd.discretize(g(dt), g(A), g(d["X"], torch.bfloat16))
    Y, F = ssd.ssd_fwd(X, la, g(d["B"], torch.bfloat16), g(d["C"], torch.bfloat16), 256, D=g(d["D"]),
                       init_states=g(d["init_states"]))
    torch.cuda.synchronize()
    la_r, X_r = oracle.discretize(dt, A, d["X"])
    # the scan reads X as the GPU rounded it: give the oracle the same values
    X_used = X.float().cpu().numpy().astype(np.float64)
    assert_close(X_used, X_r, 4e-3, "X")
    Yr, Fr = oracle.ssd_reference(X_used, la.cpu().numpy().astype(np.float64), d["B"], d["C"], d["D"],
                                  d["init_states"], None)
    assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, TAU["bf16"], "Y")
    assert_close(F.cpu().numpy().astype(np.float64), Fr, TAU["bf16"], "final states")
