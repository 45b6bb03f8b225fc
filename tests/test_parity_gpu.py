"""GPU parity of the CUDA path against the CPU fp64 oracle, through the C ABI.

Tolerance (written here, from the problem statement): over a compared tensor,
max|gpu - oracle| <= tau * max|oracle| with tau = 1e-5 for fp32 inputs and
tau = 2e-2 for bf16 inputs with fp32 state; the same rule for final states.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TAU, assert_close, run_gpu, run_oracle, slice_heads, to_device
from workloads import WORKLOADS, make_custom, make_inputs

pytestmark = pytest.mark.gpu

PATHS = ["simt", "tcgen05", "fused"]


def _ssd():
    import mamba_ssd_layer_chunked_b200 as ssd
    return ssd


def _skip_unsupported(d, dtype, chunk, path):
    ssd = _ssd()
    if path == "auto":
        return
    X = d["X"]
    p = ssd.make_problem(X.shape[0], X.shape[1], X.shape[2], X.shape[3], d["B"].shape[3], d["B"].shape[2], chunk,
                         d["nseq"], torch.bfloat16 if dtype == "bf16" else torch.float32)
    if not ssd.path_supported(p, path):
        pytest.skip(f"{path} does not cover this shape")


# --------------------------------------------------------------------------- #
# The tiny fp32 workload, in full
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("path", ["auto", "simt"])
def test_tiny_f32_workload(path):
    w = WORKLOADS["tiny_f32"]
    d = make_inputs(w)
    Y, F = run_gpu(d, w.dtype, w.chunk, path)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU["f32"], "Y")
    assert_close(F, Fr, TAU["f32"], "final_states")


# --------------------------------------------------------------------------- #
# Small cases spanning several chunks with ragged sequence pieces
# --------------------------------------------------------------------------- #

SMALL = {
    # name: (batch, T, H, P, N, G, Q, dtype, lengths, D, init)
    "bf16_varlen_N128_Q256": (2, 1024, 4, 64, 128, 1, 256, "bf16", [[100, 37, 300, 587], [1024]], "normal", True),
    "bf16_single_N64_Q128": (2, 768, 4, 64, 64, 1, 128, "bf16", None, "none", False),
    "bf16_init_N128_Q128": (1, 512, 6, 64, 128, 1, 128, "bf16", None, "normal", True),
    "bf16_N16_Q256": (1, 768, 4, 64, 16, 1, 256, "bf16", None, "none", True),
    "bf16_N256_Q256": (1, 512, 2, 64, 256, 1, 256, "bf16", [[200, 312]], "none", True),
    "bf16_groups2": (2, 512, 4, 64, 128, 2, 128, "bf16", None, "normal", False),
    "bf16_boundary_at_chunk_edge": (1, 768, 2, 64, 128, 1, 256, "bf16", [[256, 256, 256]], "none", True),
    "bf16_short_seqs": (1, 512, 2, 64, 64, 1, 256, "bf16", [[1, 1, 3, 250, 1, 256]], "normal", True),
    "f32_varlen_P32_N48_Q64": (2, 320, 3, 32, 48, 1, 64, "f32", [[1, 63, 64, 100, 92], [320]], "normal", True),
    "f32_P16_N16_Q128": (1, 384, 5, 16, 16, 1, 128, "f32", None, "ones", False),
}


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_cases(name, path):
    b, T, H, P, N, G, Q, dtype, lengths, D, init = SMALL[name]
    nseq = None if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, ngroups=G, dtype=dtype, seed=zlib.crc32(name.encode()) % 10000, has_D=D, has_init=init,
                    lengths=lengths, nseq=nseq)
    _skip_unsupported(d, dtype, Q, path)
    Y, F = run_gpu(d, dtype, Q, path)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU[dtype], "Y")
    assert_close(F, Fr, TAU[dtype], "final_states")


# --------------------------------------------------------------------------- #
# Each step on its own, against the oracle's intermediate of the same name
# --------------------------------------------------------------------------- #

STEP_CASES = ["bf16_varlen_N128_Q256", "f32_varlen_P32_N48_Q64", "bf16_single_N64_Q128"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", STEP_CASES)
def test_steps(name, path):
    ssd = _ssd()
    b, T, H, P, N, G, Q, dtype, lengths, D, init = SMALL[name]
    nseq = 1 if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, ngroups=G, dtype=dtype, seed=7 + len(name), has_D=D, has_init=init,
                    lengths=lengths, nseq=nseq if lengths else None)
    _skip_unsupported(d, dtype, Q, path)
    g = to_device(d, dtype)
    tau = TAU[dtype]
    # step 1: chunk_cumsum
    cs = ssd.chunk_cumsum(g["log_a"], Q)
    cs_ref = oracle.chunk_cumsum(d["log_a"], Q)
    assert_close(cs.cpu().numpy().astype(np.float64), cs_ref, 1e-5, "cs")
    inc_ref, loc_ref = oracle.chunk_states(d["X"], d["log_a"], d["B"], Q, d["init_states"], d["seq_idx"],
                                           nseq=nseq)
    # step 2: chunk_state (plus sequence partials)
    final = torch.zeros((b, nseq, H, N, P), dtype=torch.float32, device="cuda")
    st = ssd.chunk_state(g["X"], g["B"], cs, Q, g["seq_idx"], nseq, final_partials=final, path=path)
    assert_close(st.cpu().numpy().astype(np.float64), loc_ref, tau, "chunk_state")
    # step 3: state_passing (from the GPU chunk states)
    inc = ssd.state_passing(cs, st, tuple(g["X"].shape), N, G, Q, g["init_states"], g["seq_idx"], nseq,
                            final_states=final, dtype=g["X"].dtype)
    Yr, Fr = run_oracle(d)
    assert_close(inc.cpu().numpy().astype(np.float64), inc_ref, tau, "incoming states")
    assert_close(final.cpu().numpy().astype(np.float64), Fr, tau, "final_states")
    # state_passing alone, fed the oracle's chunk states: fp32 arithmetic
    st_ref = torch.from_numpy(np.ascontiguousarray(loc_ref, dtype=np.float32)).cuda()
    cs_ref32 = torch.from_numpy(np.ascontiguousarray(cs_ref, dtype=np.float32)).cuda()
    inc2 = ssd.state_passing(cs_ref32, st_ref, tuple(g["X"].shape), N, G, Q, g["init_states"], g["seq_idx"], nseq,
                             dtype=g["X"].dtype)
    assert_close(inc2.cpu().numpy().astype(np.float64), inc_ref, 1e-5, "incoming states (oracle inputs)")
    # step 4: chunk_scan, fed the oracle's incoming states
    Y = ssd.chunk_scan(g["X"], g["B"], g["C"], cs, torch.from_numpy(np.ascontiguousarray(inc_ref, dtype=np.float32)).cuda(), Q,
                       D=g["D"], init_states=g["init_states"], seq_idx=g["seq_idx"], nseq=nseq, path=path)
    assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, tau, "chunk_scan Y")


# --------------------------------------------------------------------------- #
# The fused path, kernel by kernel, against the oracle's quantities at segment
# level (a segment is a chunk of the block algorithm)
# --------------------------------------------------------------------------- #

FUSED_CASES = [
    # (name, seglen)
    ("bf16_varlen_N128_Q256", 256),
    ("bf16_varlen_N128_Q256", 384),   # ragged last segment
    ("bf16_single_N64_Q128", 128),
    ("bf16_short_seqs", 256),
    ("bf16_init_N128_Q128", 1024),    # one segment
    ("bf16_groups2", 256),
]


@pytest.mark.parametrize("name,seglen", FUSED_CASES)
def test_fused_steps(name, seglen):
    ssd = _ssd()
    b, T, H, P, N, G, Q, dtype, lengths, D, init = SMALL[name]
    nseq = 1 if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, ngroups=G, dtype=dtype, seed=31 + seglen, has_D=D, has_init=init,
                    lengths=lengths, nseq=nseq if lengths else None)
    _skip_unsupported(d, dtype, Q, "fused")
    g = to_device(d, dtype)
    tau = TAU[dtype]
    X, B, C = g["X"], g["B"], g["C"]
    inc_ref, loc_ref = oracle.chunk_states(d["X"], d["log_a"], d["B"], seglen, d["init_states"], d["seq_idx"],
                                           nseq=nseq)
    dec_ref = oracle.segment_decay(d["log_a"], seglen, d["seq_idx"])
    Yr, Fr = run_oracle(d)
    nseg = -(-T // seglen)
    if nseg > 1:
        st, dec = ssd.segment_state(X, g["log_a"], B, seglen, g["seq_idx"], nseq)
        assert_close(st.cpu().numpy().astype(np.float64), loc_ref, tau, "segment states")
        assert_close(dec.cpu().numpy().astype(np.float64), dec_ref, 1e-5, "segment decay")
        inc = ssd.segment_passing(st, dec, X, B, seglen, g["init_states"], g["seq_idx"], nseq)
        assert_close(inc.cpu().numpy().astype(np.float64), inc_ref, tau, "segment incoming states")
        # segment_passing alone, fed the oracle's states and decays: fp32 arithmetic
        st2 = torch.from_numpy(np.ascontiguousarray(loc_ref, dtype=np.float32)).cuda()
        dec2 = torch.from_numpy(np.ascontiguousarray(dec_ref, dtype=np.float32)).cuda()
        inc2 = ssd.segment_passing(st2, dec2, X, B, seglen, g["init_states"], g["seq_idx"], nseq)
        assert_close(inc2.cpu().numpy().astype(np.float64), inc_ref, 1e-5, "segment incoming (oracle inputs)")
        seg_in = torch.from_numpy(np.ascontiguousarray(inc_ref, dtype=np.float32)).cuda()
    else:
        seg_in = None
    # fused_scan fed the oracle's incoming segment states
    F = torch.full((b, nseq, H, N, P), float("nan"), dtype=torch.float32, device="cuda")
    Y = ssd.fused_scan(X, g["log_a"], B, C, seglen, seg_in, D=g["D"], init_states=g["init_states"],
                       seq_idx=g["seq_idx"], nseq=nseq, final_states=F)
    torch.cuda.synchronize()
    assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, tau, "fused_scan Y")
    assert_close(F.cpu().numpy().astype(np.float64), Fr, tau, "fused_scan final states")


# --------------------------------------------------------------------------- #
# Edge cases
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("path", PATHS)
def test_single_chunk(path):
    d = make_custom(2, 256, 2, 64, 128, dtype="bf16", seed=11, has_D="normal", has_init=True)
    _skip_unsupported(d, "bf16", 256, path)
    Y, F = run_gpu(d, "bf16", 256, path)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU["bf16"], "Y")
    assert_close(F, Fr, TAU["bf16"], "final")


@pytest.mark.parametrize("path", PATHS)
def test_absent_sequence_ids_keep_initial_state(path):
    d = make_custom(2, 512, 2, 64, 64, dtype="bf16", seed=12, has_init=True, lengths=[[300, 212], [512]], nseq=4)
    _skip_unsupported(d, "bf16", 128, path)
    Y, F = run_gpu(d, "bf16", 128, path)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU["bf16"], "Y")
    assert_close(F, Fr, TAU["bf16"], "final")
    np.testing.assert_array_equal(F[0, 2:], d["init_states"][0, 2:])
    np.testing.assert_array_equal(F[1, 1:], d["init_states"][1, 1:])


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("la", [0.0, -30.0])
def test_extreme_decays(path, la):
    d = make_custom(1, 512, 2, 64, 64, dtype="bf16", seed=13, has_D="normal", has_init=True)
    d["log_a"] = np.full_like(d["log_a"], la)
    _skip_unsupported(d, "bf16", 256, path)
    Y, F = run_gpu(d, "bf16", 256, path)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU["bf16"], "Y")
    assert_close(F, Fr, TAU["bf16"], "final")


def test_outputs_stay_in_bounds_and_are_deterministic():
    """Canary guard in place of a memory checker: Y and final_states are carved
    out of larger buffers whose margins hold a sentinel."""
    ssd = _ssd()
    d = make_custom(2, 512, 4, 64, 128, dtype="bf16", seed=14, has_D="normal", has_init=True,
                    lengths=[[130, 382], [512]], nseq=2)
    g = to_device(d, "bf16")
    pad = 4096
    ybuf = torch.full((g["X"].numel() + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    fbuf = torch.full((2 * 2 * 4 * 128 * 64 + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    Y = ybuf[pad:pad + g["X"].numel()].view_as(g["X"])
    F = fbuf[pad:pad + 2 * 2 * 4 * 128 * 64].view(2, 2, 4, 128, 64)
    outs = []
    for _ in range(2):
        ssd.ssd_fwd(g["X"], g["log_a"], g["B"], g["C"], 256, D=g["D"], init_states=g["init_states"],
                    seq_idx=g["seq_idx"], nseq=2, out=Y, final_out=F)
        torch.cuda.synchronize()
        outs.append((Y.clone(), F.clone()))
    for buf in (ybuf, fbuf):
        assert bool((buf[:pad] == 7.0).all()) and bool((buf[-pad:] == 7.0).all())
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    Yr, Fr = run_oracle(d)
    assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, TAU["bf16"], "Y")


def test_nondefault_stream():
    ssd = _ssd()
    d = make_custom(1, 512, 2, 64, 64, dtype="bf16", seed=15)
    g = to_device(d, "bf16")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        Y, F = ssd.ssd_fwd(g["X"], g["log_a"], g["B"], g["C"], 128)
    s.synchronize()
    Yr, Fr = run_oracle(d)
    assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, TAU["bf16"], "Y")


def test_host_buffer_entry_point():
    ssd = _ssd()
    d = make_custom(1, 512, 2, 64, 64, dtype="bf16", seed=16, has_D="normal")
    Xh = torch.from_numpy(d["X"]).to(torch.bfloat16).pin_memory()
    la = torch.from_numpy(d["log_a"]).pin_memory()
    Bh = torch.from_numpy(d["B"]).to(torch.bfloat16).pin_memory()
    Ch = torch.from_numpy(d["C"]).to(torch.bfloat16).pin_memory()
    Dh = torch.from_numpy(d["D"])
    Y, F = ssd.ssd_fwd_host(Xh, la, Bh, Ch, 128, D=Dh)
    assert not Y.is_cuda
    Yr, Fr = run_oracle(d)
    assert_close(Y.float().numpy().astype(np.float64), Yr, TAU["bf16"], "Y")
    assert_close(F.numpy().astype(np.float64), Fr, TAU["bf16"], "final")


# --------------------------------------------------------------------------- #
# Full-size workloads, in the configuration the benchmark times, on sampled
# (batch row, head) pairs the oracle computes one by one
# --------------------------------------------------------------------------- #

FULL = ["mamba2_130m_layer", "mamba2_2p7b_layer", "long16k_N16", "long16k_N64", "long16k_N128", "long16k_N256",
        "packed_varlen"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    w = WORKLOADS[name]
    d = make_inputs(w)
    Y, F = run_gpu(d, w.dtype, w.chunk, "auto")
    rng = np.random.default_rng(99)
    pairs = {(int(rng.integers(w.batch)), int(rng.integers(w.nheads))) for _ in range(6)}
    pairs |= {(0, 0), (w.batch - 1, w.nheads - 1)}
    for b, h in sorted(pairs):
        s = slice_heads(d, b, h)
        Yr, Fr = run_oracle(s)
        assert_close(Y[b:b + 1, :, h:h + 1], Yr, TAU[w.dtype], f"Y[b={b},h={h}]")
        assert_close(F[b:b + 1, :, h:h + 1], Fr, TAU[w.dtype], f"final[b={b},h={h}]")
