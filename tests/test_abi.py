"""C-ABI checks that need no GPU: the library loads, exports every function
include/ssd.h declares, and rejects bad arguments on the host before any
launch. Calls here use fake device addresses only where a host check is sure to
reject the call first, so the tests are also safe on a GPU machine."""
import ctypes
import os

import pytest

import mamba_ssd_layer_chunked_b200 as ssd
from mamba_ssd_layer_chunked_b200 import ssd as _ssd

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = range(5)
FAKE = 0x10000  # 16-byte aligned fake device address (never dereferenced here)


def prob(**kw):
    base = dict(batch=2, seqlen=512, nheads=4, headdim=64, dstate=128, ngroups=1, chunk=256, nseq=1,
                dtype=ssd.ssd.SSD_DTYPE_BF16, path=0)
    base.update(kw)
    return ssd.Problem(**base)


def test_library_exports_every_declared_function():
    names = ssd.declared_functions()
    assert "ssd_fwd" in names and "ssd_fwd_workspace_bytes" in names
    lib = ssd.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) >= {"ssd_status_string", "ssd_chunk_cumsum", "ssd_chunk_state", "ssd_state_passing",
                          "ssd_chunk_scan", "ssd_check_problem", "ssd_path_supported", "ssd_states_bytes",
                          "ssd_last_cuda_error_string", "ssd_segment_state", "ssd_segment_passing",
                          "ssd_fused_scan", "ssd_fused_work_tiles", "ssd_fused_work_count", "ssd_device_error",
                          "ssd_selftest_wait_timeout"}


def test_problem_struct_layout():
    assert ctypes.sizeof(ssd.Problem) == 8 * 8 + 2 * 4


def test_status_strings():
    for s, text in [(OK, "ok"), (INVALID, "invalid argument"), (WORKSPACE, "workspace missing or too small"),
                    (5, "a device-side wait gave up (outputs invalid)")]:
        assert ssd.status_string(s) == text
    assert ssd.status_string(99) == "unknown status"


def test_workspace_bytes_formula():
    p = prob()
    align = lambda x: (x + 255) // 256 * 256
    cs = 2 * 512 * 4 * 4  # cumsum values x 4 bytes; the SIMT family keeps them in fp64 (x 2)
    st = 2 * (512 // 256) * 4 * 128 * 64 * 4
    # fused: rows (batch, head pair) = 4, 4 tiles each; ranges of wt tiles
    wt = ssd.fused_work_tiles(p)
    total = 2 * 2 * 4
    assert 1 <= wt <= total  # about one range per SM of the device (or of a 148-SM part without one)
    nwork = -(-total // wt)
    assert ssd.fused_work_count(p, wt) == nwork
    fused = 2 * align(nwork * 2 * 128 * 64 * 4) + align(nwork * 2 * 4)
    assert ssd.workspace_bytes(p) == fused  # AUTO runs the fused family for this problem
    assert ssd.workspace_bytes(prob(path=1)) == align(2 * cs) + align(st)  # the SIMT family: the chunked need
    # value 2 of ssd_path (the retired chunked tensor-core family) is not a path
    assert ssd.lib().ssd_fwd_workspace_bytes(ctypes.byref(prob(path=2))) == ctypes.c_size_t(-1).value
    assert ssd.lib().ssd_check_problem(ctypes.byref(prob(path=2))) == INVALID
    assert ssd.states_bytes(p) == st
    # outside the fused domain (fp32) only the chunked need counts
    q = prob(dtype=ssd.ssd.SSD_DTYPE_F32)
    assert ssd.fused_work_tiles(q) == -1
    assert ssd.workspace_bytes(q) == align(2 * cs) + align(st)


def test_fused_work_count():
    p = prob()  # 16 tiles in all
    assert ssd.fused_work_count(p, 3) == 6
    assert ssd.fused_work_count(p, 16) == 1
    for bad in (0, -2, 17):
        assert ssd.fused_work_count(p, bad) == -1


@pytest.mark.parametrize("field,value,expect", [
    ("batch", 0, INVALID), ("seqlen", 0, INVALID), ("nheads", 0, INVALID), ("headdim", -1, INVALID),
    ("dstate", 0, INVALID), ("ngroups", 3, INVALID), ("nseq", 0, INVALID), ("dtype", 7, INVALID),
    ("path", 9, INVALID), ("chunk", 100, UNSUPPORTED),
    ("headdim", 24, UNSUPPORTED), ("dstate", 512, UNSUPPORTED)])
def test_bad_problem_rejected(field, value, expect):
    p = prob(**{field: value})
    lib = ssd.lib()
    assert lib.ssd_fwd_workspace_bytes(ctypes.byref(p)) == ctypes.c_size_t(-1).value
    assert lib.ssd_check_problem(ctypes.byref(p)) == expect
    assert lib.ssd_fwd(ctypes.byref(p), *([FAKE] * 9), FAKE, 1 << 30, None) == expect


def test_ragged_length_is_supported_by_every_family():
    # T % Q != 0: the last chunk is partial (host-side sizes only; the GPU
    # parity tests run ragged lengths on every family). No call reaches a launch.
    lib = ssd.lib()
    p = prob(seqlen=500)  # bf16, P 64, N 128
    f = prob(seqlen=500, dtype=ssd.ssd.SSD_DTYPE_F32)  # fp32: the SIMT family
    assert lib.ssd_check_problem(ctypes.byref(f)) in (OK, UNSUPPORTED)  # UNSUPPORTED only without a B200
    nchunks = -(-500 // 256)
    assert lib.ssd_states_bytes(ctypes.byref(f)) == 2 * nchunks * 4 * 128 * 64 * 4
    assert ssd.workspace_bytes(p) > 0 and ssd.workspace_bytes(f) > 0


def test_null_problem_rejected():
    lib = ssd.lib()
    assert lib.ssd_check_problem(None) == INVALID
    assert lib.ssd_fwd(None, *([FAKE] * 9), FAKE, 1 << 30, None) == INVALID


def _fwd(p, X=FAKE, la=FAKE, B=FAKE, C=FAKE, D=None, init=None, seq=None, Y=FAKE, fin=None, ws=FAKE,
         wsb=1 << 30):
    return ssd.lib().ssd_fwd(ctypes.byref(p), X, la, B, C, D, init, seq, Y, fin, ws, wsb, None)


@pytest.mark.parametrize("arg", ["X", "la", "B", "C", "Y"])
def test_null_required_pointer(arg):
    assert _fwd(prob(), **{arg: None}) == INVALID


@pytest.mark.parametrize("arg", ["X", "la", "B", "C", "D", "init", "seq", "Y", "fin", "ws"])
def test_misaligned_pointer(arg):
    # 16-byte alignment, except log a, D and seq_idx: 4-byte (read one element at a time)
    p = prob(nseq=2) if arg == "seq" else prob()
    assert _fwd(p, **{arg: FAKE + (2 if arg in ("la", "D", "seq") else 4)}) == INVALID


def test_nseq_needs_seq_idx():
    assert _fwd(prob(nseq=3)) == INVALID


def test_sp_summary_workspace_formula():
    lib = ssd.lib()
    align = lambda x: (x + 255) // 256 * 256
    size = lambda q: lib.ssd_sp_summary_workspace_bytes(ctypes.byref(q))
    # segment_state covers bf16, P 64, N 64 or 128: no workspace
    assert size(prob()) == 0 and size(prob(dstate=64)) == 0
    # the chunked steps: cumsum (fp64), chunk states, final states from zero
    for q, (b, T, H, P, N, Q, S, csb) in ((prob(dtype=ssd.ssd.SSD_DTYPE_F32, headdim=16, dstate=16, chunk=64),
                                           (2, 512, 4, 16, 16, 64, 1, 8)),
                                          (prob(dstate=256), (2, 512, 4, 64, 256, 256, 1, 8)),
                                          (prob(seqlen=500, nseq=3, path=1), (2, 500, 4, 64, 128, 256, 3, 8)),
                                          (prob(path=1), (2, 512, 4, 64, 128, 256, 1, 8))):
        nc = -(-T // Q)
        want = align(b * nc * Q * H * csb) + align(b * nc * H * N * P * 4) + align(b * S * H * N * P * 4)
        assert size(q) == want
    assert size(prob(batch=0)) == ctypes.c_size_t(-1).value


def test_workspace_checks():
    p = prob()
    need = ssd.workspace_bytes(p)
    assert _fwd(p, ws=None) == WORKSPACE
    assert _fwd(p, wsb=need - 1) == WORKSPACE


def test_step_entry_points_validate_on_host():
    lib = ssd.lib()
    p = prob()
    assert lib.ssd_chunk_cumsum(ctypes.byref(p), None, FAKE, None) == INVALID
    assert lib.ssd_chunk_cumsum(ctypes.byref(p), FAKE + 2, FAKE, None) == INVALID  # log a: 4-byte
    assert lib.ssd_chunk_cumsum(ctypes.byref(p), FAKE, FAKE + 8, None) == INVALID  # cs: 16-byte
    assert lib.ssd_chunk_state(ctypes.byref(p), None, FAKE, FAKE, None, FAKE, None, None) == INVALID
    assert lib.ssd_state_passing(ctypes.byref(p), FAKE, None, FAKE, None, None, None, None) == INVALID
    assert lib.ssd_chunk_scan(ctypes.byref(p), FAKE, FAKE, None, FAKE, None, FAKE, None, None, FAKE,
                              None) == INVALID
    q = prob(nseq=2)
    assert lib.ssd_state_passing(ctypes.byref(q), FAKE, FAKE, FAKE, None, None, None, None) == INVALID
    # fused steps: bad work range lengths and null pointers are rejected on the host
    for wt in (0, -1, 17):
        assert lib.ssd_segment_state(ctypes.byref(p), wt, FAKE, FAKE, FAKE, None, FAKE, FAKE, None) == INVALID
        assert lib.ssd_segment_passing(ctypes.byref(p), wt, FAKE, FAKE, None, None, FAKE, None) == INVALID
        assert lib.ssd_fused_scan(ctypes.byref(p), wt, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None, FAKE, None,
                                  None) == INVALID
    assert lib.ssd_segment_state(ctypes.byref(p), 3, None, FAKE, FAKE, None, FAKE, FAKE, None) == INVALID
    assert lib.ssd_segment_passing(ctypes.byref(p), 3, FAKE, FAKE, None, None, None, None) == INVALID
    assert lib.ssd_fused_scan(ctypes.byref(p), 3, FAKE, FAKE, FAKE, FAKE, None, None, None, None, FAKE, None,
                              None) == INVALID  # ranges that start inside a row need the incoming states


def test_binding_rejects_host_tensors_and_bad_shapes():
    import torch
    X = torch.zeros(1, 256, 2, 16)
    la = torch.zeros(1, 256, 2)
    B = torch.zeros(1, 256, 1, 16)
    with pytest.raises(ValueError):
        _ssd._check_shapes(X, la[:, :, :1], B, B, None, None, None, 1)
    with pytest.raises(TypeError):
        _ssd._check_shapes(X.double(), la, B.double(), B.double(), None, None, None, 1)
    with pytest.raises(ValueError):
        _ssd._ptr(X)  # CPU tensor


def test_sequence_parallel_entry_points_validate_on_host():
    lib = ssd.lib()
    p = prob()
    # summary: every pointer is required, 16-byte alignment
    summ = lambda q, *a: lib.ssd_sp_summary(ctypes.byref(q), *a)
    assert summ(p, None, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, 0, None) == INVALID
    assert summ(p, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None, 0, None) == INVALID
    assert summ(p, FAKE + 8, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, 0, None) == INVALID
    assert summ(prob(nseq=2), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, 0, None) == INVALID  # needs seq_idx
    # outside the fused kernels' domain the chunked steps need a workspace
    q = prob(dtype=ssd.ssd.SSD_DTYPE_F32, headdim=16, dstate=16, chunk=64)
    need = lib.ssd_sp_summary_workspace_bytes(ctypes.byref(q))
    assert summ(q, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, 0, None) == WORKSPACE
    assert summ(q, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, need - 1, None) == WORKSPACE
    assert summ(q, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE + 8, need, None) == INVALID
    # combine and ownership: rank within [0, nranks), buffers present
    for nranks, rank in ((0, 0), (2, 2), (2, -1)):
        assert lib.ssd_sp_combine(ctypes.byref(p), nranks, rank, FAKE, FAKE, FAKE, None, FAKE, None) == INVALID
        assert lib.ssd_sp_own_finals(ctypes.byref(p), nranks, rank, FAKE, FAKE, None) == INVALID
    assert lib.ssd_sp_combine(ctypes.byref(p), 2, 1, None, FAKE, FAKE, None, FAKE, None) == INVALID
    assert lib.ssd_sp_combine(ctypes.byref(p), 2, 1, FAKE, FAKE, FAKE, None, None, None) == INVALID
    assert lib.ssd_sp_own_finals(ctypes.byref(p), 2, 1, None, FAKE, None) == INVALID
    assert lib.ssd_sp_own_finals(ctypes.byref(p), 2, 1, FAKE, FAKE + 4, None) == INVALID


def test_header_is_plain_c_and_a_c_program_links(tmp_path):
    """include/ssd.h compiles as C99 and a C program links against the library
    and calls its host-only functions (no device needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use.c"
    src.write_text(
        '#include <stdio.h>\n#include "ssd.h"\n'
        "int main(void) {\n"
        "    ssd_problem p = {2, 512, 4, 64, 128, 1, 256, 1, SSD_DTYPE_BF16, SSD_PATH_SIMT};\n"
        '    printf("%s %zu %zu\\n", ssd_status_string(SSD_OK), ssd_fwd_workspace_bytes(&p), ssd_states_bytes(&p));\n'
        "    return ssd_check_problem(NULL) == SSD_ERR_INVALID_ARG ? 0 : 1;\n}\n")
    lib_dir = os.path.dirname(ssd.ssd.LIB_PATH)
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"), str(src),
                    "-o", str(exe), ssd.ssd.LIB_PATH, "-Wl,-rpath," + lib_dir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    align = lambda x: (x + 255) // 256 * 256
    st = 2 * 2 * 4 * 128 * 64 * 4
    assert out == ["ok", str(align(2 * 2 * 512 * 4 * 4) + align(st)), str(st)]
