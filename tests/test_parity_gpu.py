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
from gpu_util import TAU, assert_close, run_gpu, run_oracle, to_device
from workloads import WORKLOADS, make_custom, make_inputs

pytestmark = pytest.mark.gpu

PATHS = ["simt", "fused"]


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
    # one head per group, and an odd number of heads per group (outside the fused family's pairs)
    "bf16_group_per_head": (1, 512, 4, 64, 64, 4, 128, "bf16", [[300, 212]], "normal", True),
    "bf16_three_heads_per_group": (1, 640, 6, 64, 128, 2, 256, "bf16", None, "normal", True),
    "f32_groups3_P32": (2, 256, 6, 32, 32, 3, 64, "f32", [[100, 156], [256]], "normal", True),
    "bf16_boundary_at_chunk_edge": (1, 768, 2, 64, 128, 1, 256, "bf16", [[256, 256, 256]], "none", True),
    "bf16_short_seqs": (1, 512, 2, 64, 64, 1, 256, "bf16", [[1, 1, 3, 250, 1, 256]], "normal", True),
    "f32_varlen_P32_N48_Q64": (2, 320, 3, 32, 48, 1, 64, "f32", [[1, 63, 64, 100, 92], [320]], "normal", True),
    "bf16_ragged_tile_Q64": (2, 576, 4, 64, 128, 1, 64, "bf16", [[200, 376], [576]], "normal", True),
    # T not a multiple of Q (or of the 128-token tile)
    "bf16_ragged_T1000_Q256": (2, 1000, 4, 64, 128, 1, 256, "bf16", [[400, 600], [1000]], "normal", True),
    # ids that never occur (zero-length sequences): they keep their initial state
    "bf16_skipped_ids_Q128": (2, 512, 4, 64, 128, 1, 128, "bf16", [[100, 0, 300, 0, 112], [512, 0, 0, 0, 0]],
                              "normal", True),
    "f32_skipped_ids_Q64": (2, 256, 3, 32, 48, 1, 64, "f32", [[60, 0, 100, 96], [0, 256, 0, 0]], "normal", True),
    "f32_P16_N16_Q128": (1, 384, 5, 16, 16, 1, 128, "f32", None, "ones", False),
    # partial last chunks on the chunked families too
    "f32_ragged_T300_Q64": (2, 300, 3, 32, 48, 1, 64, "f32", [[100, 200], [300]], "normal", True),
    "f32_ragged_T70_Q128": (1, 70, 2, 16, 16, 1, 128, "f32", None, "ones", True),
    "bf16_ragged_boundary_in_last_chunk": (1, 700, 4, 64, 128, 1, 256, "bf16", [[600, 100]], "normal", True),
    # head dimension 128: one head per row of the fused family, its two 64-column halves as the slots
    "bf16_P128_varlen_N128": (2, 900, 3, 128, 128, 1, 256, "bf16", [[250, 650], [900]], "normal", True),
    "bf16_P128_groups2_N64": (1, 640, 4, 128, 64, 2, 128, "bf16", None, "normal", False),
    "bf16_P128_N256_slices": (1, 512, 2, 128, 256, 1, 256, "bf16", [[200, 312]], "normal", True),
    # an odd number of heads per group with ranges that cut rows (the half-empty last pair)
    "bf16_odd_heads_varlen": (2, 1500, 5, 64, 128, 1, 256, "bf16", [[700, 800], [1500]], "normal", True),
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


@pytest.mark.parametrize("path", ["simt"])  # the chunked steps run on the SIMT kernels
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
# The fused path, kernel by kernel, against the oracle's states at the cuts of
# the work ranges (a range's piece of a row is a block of the block algorithm)
# --------------------------------------------------------------------------- #

FUSED_CASES = [
    # (name, work_tiles)
    ("bf16_varlen_N128_Q256", 3),     # ranges start and end inside rows and span rows
    ("bf16_varlen_N128_Q256", 5),
    ("bf16_varlen_N128_Q256", 8),     # one range per row: no cut inside a row
    ("bf16_varlen_N128_Q256", 32),    # one range for everything
    ("bf16_single_N64_Q128", 4),
    ("bf16_single_N64_Q128", 7),
    ("bf16_short_seqs", 1),           # one tile per range
    ("bf16_short_seqs", 3),
    ("bf16_init_N128_Q128", 5),
    ("bf16_groups2", 3),
    ("bf16_boundary_at_chunk_edge", 2),  # cuts on sequence boundaries
    ("bf16_ragged_tile_Q64", 3),      # a short last tile in every row
    ("bf16_ragged_T1000_Q256", 3),    # T not a multiple of the chunk
]


def _cut_states(d, wt, nseq):
    """The oracle's (local, decay, incoming) at the cuts of the work ranges,
    [nwork, 2, N, P] / [nwork, 2] / [nwork, 2, N, P], NaN where not defined:
    local/decay for ranges whose last piece ends inside its row, incoming for
    ranges whose first piece starts inside its row. Each is the oracle's
    per-block quantity on a slice of the row: the slice [s0, s1) as one block
    for the local state and decay, and [0, s0 + 1) cut at s0 for the incoming state."""
    X, la, B, init, seq = d["X"], d["log_a"], d["B"], d["init_states"], d["seq_idx"]
    b, T, H, P = X.shape
    N = B.shape[3]
    npairs, nt = H // 2, -(-T // 128)
    total = b * npairs * nt
    nwork = -(-total // wt)
    loc = np.full((nwork, 2, N, P), np.nan)
    dec = np.full((nwork, 2), np.nan)
    inc = np.full((nwork, 2, N, P), np.nan)
    sl_seq = lambda bb, a, e: None if seq is None else seq[bb:bb + 1, a:e]
    for i in range(nwork):
        fb, fe = i * wt, min((i + 1) * wt, total)
        r = (fe - 1) // nt
        s0, s1 = 128 * max(fb - r * nt, 0), min(128 * (fe - r * nt), T)
        bb, hp = divmod(r, npairs)
        hs = slice(2 * hp, 2 * hp + 2)
        if s1 < T:
            _, lo = oracle.chunk_states(X[bb:bb + 1, s0:s1], la[bb:bb + 1, s0:s1], B[bb:bb + 1, s0:s1], s1 - s0,
                                        None, sl_seq(bb, s0, s1), nseq=nseq)
            loc[i] = lo[0, 0, hs]
            dec[i] = oracle.segment_decay(la[bb:bb + 1, s0:s1], s1 - s0, sl_seq(bb, s0, s1))[0, 0, hs]
        r0 = fb // nt
        s0 = 128 * (fb - r0 * nt)
        if s0 > 0:
            bb, hp = divmod(r0, npairs)
            hs = slice(2 * hp, 2 * hp + 2)
            ini = None if init is None else init[bb:bb + 1]
            ic, _ = oracle.chunk_states(X[bb:bb + 1, :s0 + 1], la[bb:bb + 1, :s0 + 1], B[bb:bb + 1, :s0 + 1], s0,
                                        ini, sl_seq(bb, 0, s0 + 1), nseq=nseq)
            inc[i] = ic[0, 1, hs]
    return loc, dec, inc


def _close_where(got, ref, tau, what, atol=0.0):
    m = ~np.isnan(ref)
    assert m.any(), what
    assert_close(got[m], ref[m], tau, what, atol)


@pytest.mark.parametrize("name,wt", FUSED_CASES)
def test_fused_steps(name, wt):
    ssd = _ssd()
    b, T, H, P, N, G, Q, dtype, lengths, D, init = SMALL[name]
    nseq = 1 if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, ngroups=G, dtype=dtype, seed=31 + wt, has_D=D, has_init=init,
                    lengths=lengths, nseq=nseq if lengths else None)
    _skip_unsupported(d, dtype, Q, "fused")
    g = to_device(d, dtype)
    tau = TAU[dtype]
    X, B, C = g["X"], g["B"], g["C"]
    Yr, Fr = run_oracle(d)
    nt = -(-T // 128)
    nwork = -(-(b * (H // 2) * nt) // wt)
    p = ssd.make_problem(b, T, H, P, N, G, Q, nseq, torch.bfloat16, path="fused")
    assert ssd.fused_work_count(p, wt) == nwork
    if nwork > 1 and wt % nt != 0:
        loc_ref, dec_ref, inc_ref = _cut_states(d, wt, nseq)
        loc, dec = ssd.segment_state(X, g["log_a"], B, wt, g["seq_idx"], nseq)
        _close_where(loc.cpu().numpy().astype(np.float64), loc_ref, tau, "range end states")
        # decays below fp32's normal range come back as 0: an absolute floor far below anything they scale
        _close_where(dec.cpu().numpy().astype(np.float64), dec_ref, 1e-5, "range decays", atol=1e-30)
        inc = ssd.segment_passing(loc, dec, X, B, wt, g["init_states"], g["seq_idx"], nseq)
        _close_where(inc.cpu().numpy().astype(np.float64), inc_ref, tau, "range incoming states")
        # segment_passing alone, fed the oracle's states and decays: fp32 arithmetic
        loc2 = torch.from_numpy(np.ascontiguousarray(loc_ref, dtype=np.float32)).cuda()
        dec2 = torch.from_numpy(np.ascontiguousarray(dec_ref, dtype=np.float32)).cuda()
        inc2 = ssd.segment_passing(loc2, dec2, X, B, wt, g["init_states"], g["seq_idx"], nseq)
        _close_where(inc2.cpu().numpy().astype(np.float64), inc_ref, 1e-5, "range incoming (oracle inputs)")
        work_in = torch.from_numpy(np.ascontiguousarray(inc_ref, dtype=np.float32)).cuda()
    else:
        loc = dec = inc = None
        work_in = None
    # fused_scan fed the oracle's incoming range states
    F = torch.full((b, nseq, H, N, P), float("nan"), dtype=torch.float32, device="cuda")
    Y = ssd.fused_scan(X, g["log_a"], B, C, wt, work_in, D=g["D"], init_states=g["init_states"],
                       seq_idx=g["seq_idx"], nseq=nseq, final_states=F)
    torch.cuda.synchronize()
    assert_close(Y.float().cpu().numpy().astype(np.float64), Yr, tau, "fused_scan Y")
    assert_close(F.cpu().numpy().astype(np.float64), Fr, tau, "fused_scan final states")
    # the chained scan (the cuts chained inside it, as ssd_fwd runs it) gives what
    # segment_passing + fused_scan give: the same fp32 chain in the same order
    F1 = torch.full_like(F, float("nan"))
    Y1 = ssd.fused_scan(X, g["log_a"], B, C, wt, inc, D=g["D"], init_states=g["init_states"],
                        seq_idx=g["seq_idx"], nseq=nseq, final_states=F1)
    F2 = torch.full_like(F, float("nan"))
    Y2 = ssd.fused_scan_chained(X, g["log_a"], B, C, wt, loc, dec, D=g["D"], init_states=g["init_states"],
                                seq_idx=g["seq_idx"], nseq=nseq, final_states=F2)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2), "chained scan Y differs from segment_passing + fused_scan"
    assert torch.equal(F1.nan_to_num(7.0), F2.nan_to_num(7.0)), "chained scan final states differ"
    assert_close(Y2.float().cpu().numpy().astype(np.float64), Yr, tau, "fused_scan_chained Y")


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
@pytest.mark.parametrize("T, dtype, P, N, Q", [(1, "bf16", 64, 128, 256), (7, "f32", 32, 48, 64),
                                              (127, "bf16", 64, 64, 128), (129, "bf16", 64, 128, 128)])
def test_single_token_and_short_rows(path, T, dtype, P, N, Q):
    # one token, and rows shorter than (or one token past) a chunk and a 128-token tile
    d = make_custom(2, T, 4, P, N, dtype=dtype, seed=14 + T, has_D="normal", has_init=True)
    _skip_unsupported(d, dtype, Q, path)
    Y, F = run_gpu(d, dtype, Q, path)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU[dtype], "Y")
    assert_close(F, Fr, TAU[dtype], "final")


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
# Full-size workloads, in the launch configuration the benchmark times, compared
# with the oracle element by element over the whole Y and final-state tensors
# --------------------------------------------------------------------------- #

FULL = ["mamba2_130m_layer", "mamba2_2p7b_layer", "long16k_N16", "long16k_N64", "long16k_N128", "long16k_N256",
        "packed_varlen"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_whole_tensor(name):
    w = WORKLOADS[name]
    d = make_inputs(w)
    Y, F = run_gpu(d, w.dtype, w.chunk, "auto")
    Yr, Fr = run_oracle(d)  # every (batch row, head), all host cores
    assert_close(Y, Yr, TAU[w.dtype], f"Y ({name})")
    assert_close(F, Fr, TAU[w.dtype], f"final_states ({name})")


# --------------------------------------------------------------------------- #
# segment_state stops its backward walk once the decay over the rest of the
# piece is below e^-40 (those terms reach the cut scaled by < 4.3e-18). Put the
# largest inputs exactly there: 2^40 times the rest, in the tiles the walk
# skips, with a cut inside the row; the outputs after the cut must still match
# the oracle to the tolerance relative to their own magnitude.
# --------------------------------------------------------------------------- #

def test_segment_walk_cut_with_large_early_inputs():
    ssd = _ssd()
    T, wt, cut = 8192, 40, 40 * 128  # ranges [0, 40) and [40, 64) of one row: a cut at token 5120
    d = make_custom(1, T, 2, 64, 128, dtype="bf16", seed=404, has_D="normal", has_init=True)
    d["log_a"] = np.full_like(d["log_a"], -0.04)  # the walk stops ~8 tiles back from the cut
    big = 30 * 128
    d["X"] = d["X"].copy()
    d["X"][:, :big] *= 2.0 ** 40  # exact in bf16: a power of two
    g = to_device(d, "bf16")
    loc, dec = ssd.segment_state(g["X"], g["log_a"], g["B"], wt)
    torch.cuda.synchronize()
    assert float(dec[0].abs().max()) == 0.0, "the walk did not stop early: the case does not exercise the cut"
    F = torch.full((1, 1, 2, 128, 64), float("nan"), dtype=torch.float32, device="cuda")
    Yg = ssd.fused_scan_chained(g["X"], g["log_a"], g["B"], g["C"], wt, loc, dec, D=g["D"],
                                init_states=g["init_states"], final_states=F)
    torch.cuda.synchronize()
    ssd.check_device_error()
    Y = Yg.float().cpu().numpy().astype(np.float64)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU["bf16"], "Y")
    assert_close(Y[:, cut:], Yr[:, cut:], TAU["bf16"], "Y after the cut (its own scale)")
    assert_close(F.cpu().numpy().astype(np.float64), Fr, TAU["bf16"], "final_states")
