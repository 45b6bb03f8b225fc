"""Python binding of libssd_b200.so (the C ABI of include/ssd.h).

Argument marshalling only: shapes and dtypes are read from torch tensors,
outputs and the workspace are allocated with torch (device memory is the
caller's, as the C ABI requires), and every step of the computation runs in
the library's CUDA kernels on the current torch stream. There is no CPU or
PyTorch fallback: if the library is missing or cannot run, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "ssd.h")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_WORKSPACE, SSD_ERR_CUDA, SSD_ERR_DEVICE_TIMEOUT = range(6)
SSD_DTYPE_F32, SSD_DTYPE_BF16 = 0, 1
PATHS = {"auto": 0, "simt": 1, "fused": 3}


class SSDError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {status_string(status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class Problem(ctypes.Structure):
    """Mirror of ssd_problem."""

    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("chunk", ctypes.c_int64), ("nseq", ctypes.c_int64), ("dtype", ctypes.c_int),
                ("path", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def _declare(lib):
    vp, P = ctypes.c_void_p, ctypes.POINTER(Problem)
    sig = {
        "ssd_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "ssd_last_cuda_error_string": ([], ctypes.c_char_p),
        "ssd_check_problem": ([P], ctypes.c_int),
        "ssd_path_supported": ([P, ctypes.c_int], ctypes.c_int),
        "ssd_fwd_workspace_bytes": ([P], ctypes.c_size_t),
        "ssd_states_bytes": ([P], ctypes.c_size_t),
        "ssd_fwd": ([P] + [vp] * 9 + [vp, ctypes.c_size_t, vp], ctypes.c_int),
        "ssd_chunk_cumsum": ([P, vp, vp, vp], ctypes.c_int),
        "ssd_chunk_state": ([P, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "ssd_state_passing": ([P, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "ssd_chunk_scan": ([P] + [vp] * 9 + [vp], ctypes.c_int),
        "ssd_fused_work_tiles": ([P], ctypes.c_int64),
        "ssd_fused_work_count": ([P, ctypes.c_int64], ctypes.c_int64),
        "ssd_segment_state": ([P, ctypes.c_int64] + [vp] * 7, ctypes.c_int),
        "ssd_segment_passing": ([P, ctypes.c_int64] + [vp] * 6, ctypes.c_int),
        "ssd_fused_scan": ([P, ctypes.c_int64] + [vp] * 11, ctypes.c_int),
        "ssd_fused_scan_chained": ([P, ctypes.c_int64] + [vp] * 12, ctypes.c_int),
        "ssd_decode_step": ([P] + [vp] * 8, ctypes.c_int),
        "ssd_discretize": ([P, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp], ctypes.c_int),
        "ssd_sp_summary": ([P] + [vp] * 8 + [ctypes.c_size_t, vp], ctypes.c_int),
        "ssd_sp_summary_workspace_bytes": ([P], ctypes.c_size_t),
        "ssd_sp_combine": ([P, ctypes.c_int, ctypes.c_int] + [vp] * 6, ctypes.c_int),
        "ssd_sp_own_finals": ([P, ctypes.c_int, ctypes.c_int, vp, vp, vp], ctypes.c_int),
        "ssd_device_error": ([ctypes.POINTER(ctypes.c_uint32), vp], ctypes.c_int),
        "ssd_selftest_wait_timeout": ([ctypes.c_uint64, vp], ctypes.c_int),
    }
    for name, (argtypes, restype) in sig.items():
        f = getattr(lib, name)
        f.argtypes = argtypes
        f.restype = restype


def lib():
    """The loaded library; raises ImportError when it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with `python mamba_ssd_layer_chunked_b200/build.py` "
                    "(there is no fallback implementation)")
            l = ctypes.CDLL(LIB_PATH)
            _declare(l)
            _lib = l
    return _lib


def declared_functions() -> list:
    """Names of the functions include/ssd.h declares (for the export check)."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().ssd_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != SSD_OK:
        detail = lib().ssd_last_cuda_error_string().decode() if status == SSD_ERR_CUDA else ""
        raise SSDError(status, what, detail)


def make_problem(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, nseq=1,
                 dtype: torch.dtype = torch.bfloat16, path: str = "auto") -> Problem:
    if dtype == torch.float32:
        dt = SSD_DTYPE_F32
    elif dtype == torch.bfloat16:
        dt = SSD_DTYPE_BF16
    else:
        raise TypeError(f"unsupported dtype {dtype} (float32 or bfloat16)")
    return Problem(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, nseq, dt, PATHS[path])


def problem_from(X: torch.Tensor, B: torch.Tensor, chunk: int, nseq: int = 1, path: str = "auto") -> Problem:
    batch, seqlen, nheads, headdim = X.shape
    ngroups, dstate = B.shape[2], B.shape[3]
    return make_problem(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, nseq, X.dtype, path)


def workspace_bytes(p: Problem) -> int:
    n = lib().ssd_fwd_workspace_bytes(ctypes.byref(p))
    if n == ctypes.c_size_t(-1).value:
        _check(lib().ssd_check_problem(ctypes.byref(p)) or SSD_ERR_INVALID_ARG, "ssd_fwd_workspace_bytes")
    return int(n)


def states_bytes(p: Problem) -> int:
    return int(lib().ssd_states_bytes(ctypes.byref(p)))


def path_supported(p: Problem, path: str) -> bool:
    return bool(lib().ssd_path_supported(ctypes.byref(p), PATHS[path]))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def device_error(stream=None) -> int:
    """Read and clear the library's device error word (synchronises `stream`):
    0 when no bounded wait of a kernel has given up since the last read; else
    the word's bits (the outputs of the calls since then are invalid)."""
    code = ctypes.c_uint32(0)
    st = lib().ssd_device_error(ctypes.byref(code), _stream(stream))
    if st not in (SSD_OK, SSD_ERR_DEVICE_TIMEOUT):
        _check(st, "ssd_device_error")
    return int(code.value)


def check_device_error(stream=None):
    """Raise SSDError when a kernel's bounded wait gave up since the last read."""
    code = device_error(stream)
    if code:
        raise SSDError(SSD_ERR_DEVICE_TIMEOUT, "ssd_device_error", f"error word 0x{code:x}")


def selftest_wait_timeout(limit_ns: int, stream=None):
    """Launch the self-test kernel whose one wait gives up after limit_ns."""
    _check(lib().ssd_selftest_wait_timeout(int(limit_ns), _stream(stream)), "ssd_selftest_wait_timeout")


def _check_shapes(X, log_a, B, C, D, init_states, seq_idx, nseq):
    if X.dim() != 4 or B.dim() != 4 or C.shape != B.shape or log_a.shape != X.shape[:3]:
        raise ValueError("shapes: X [b,T,H,P], log_a [b,T,H], B and C [b,T,G,N]")
    if B.shape[:2] != X.shape[:2]:
        raise ValueError("B and C must have the batch and sequence sizes of X")
    if X.dtype not in (torch.float32, torch.bfloat16) or B.dtype != X.dtype or C.dtype != X.dtype:
        raise TypeError("X, B and C must share one dtype, float32 or bfloat16")
    if log_a.dtype != torch.float32:
        raise TypeError("log_a must be float32")
    if D is not None and (D.dtype != torch.float32 or D.shape != (X.shape[2],)):
        raise ValueError("D must be float32 [nheads]")
    b, T, H, P = X.shape
    N = B.shape[3]
    if init_states is not None and (init_states.dtype != torch.float32 or
                                    init_states.shape != (b, nseq, H, N, P)):
        raise ValueError(f"init_states must be float32 [{b}, {nseq}, {H}, {N}, {P}]")
    if seq_idx is not None and (seq_idx.dtype != torch.int32 or seq_idx.shape != (b, T)):
        raise ValueError("seq_idx must be int32 [batch, seqlen]")


def ssd_fwd(X: torch.Tensor, log_a: torch.Tensor, B: torch.Tensor, C: torch.Tensor, chunk: int,
            D: Optional[torch.Tensor] = None, init_states: Optional[torch.Tensor] = None,
            seq_idx: Optional[torch.Tensor] = None, nseq: Optional[int] = None,
            return_final_states: bool = True, path: str = "auto",
            out: Optional[torch.Tensor] = None, final_out: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None
            ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """SSD forward on the GPU: Y [b,T,H,P] (dtype of X) and final states
    [b, nseq, H, N, P] fp32 (None unless return_final_states).

    ``nseq`` defaults to 1 without seq_idx. With seq_idx it must be given (the
    library never reads seq_idx on the host).
    """
    if nseq is None:
        if seq_idx is not None:
            raise ValueError("nseq is required with seq_idx (the number of sequences per row)")
        nseq = 1
    _check_shapes(X, log_a, B, C, D, init_states, seq_idx, nseq)
    p = problem_from(X, B, chunk, nseq, path)
    b, T, H, P = X.shape
    N = B.shape[3]
    Y = out if out is not None else torch.empty_like(X)
    final = None
    if return_final_states:
        final = final_out if final_out is not None else torch.empty((b, nseq, H, N, P), dtype=torch.float32,
                                                                   device=X.device)
    need = workspace_bytes(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    st = lib().ssd_fwd(ctypes.byref(p), _ptr(X), _ptr(log_a), _ptr(B), _ptr(C), _ptr(D), _ptr(init_states),
                       _ptr(seq_idx), _ptr(Y), _ptr(final), _ptr(workspace),
                       workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ssd_fwd")
    return Y, final


def ssd_fwd_host(X: torch.Tensor, log_a: torch.Tensor, B: torch.Tensor, C: torch.Tensor, chunk: int,
                 D=None, init_states=None, seq_idx=None, nseq=None, return_final_states=True,
                 path="auto", device="cuda", stream=None):
    """End-to-end call on HOST tensors: copy the inputs to the device (pinned
    host memory gives asynchronous copies), run ssd_fwd, copy Y (and the final
    states) back into host tensors. Returns host tensors."""
    dev = torch.device(device)
    args = [None if t is None else t.to(dev, non_blocking=True) for t in (X, log_a, B, C, D, init_states, seq_idx)]
    Y, final = ssd_fwd(*args[:4], chunk, D=args[4], init_states=args[5], seq_idx=args[6], nseq=nseq,
                       return_final_states=return_final_states, path=path, stream=stream)
    pin = X.is_pinned()
    Yh = torch.empty(Y.shape, dtype=Y.dtype, pin_memory=pin)
    Yh.copy_(Y, non_blocking=True)
    Fh = None
    if final is not None:
        Fh = torch.empty(final.shape, dtype=final.dtype, pin_memory=pin)
        Fh.copy_(final, non_blocking=True)
    torch.cuda.current_stream(dev).synchronize()
    return Yh, Fh


# ---- the four steps, one call each -----------------------------------------

def chunk_cumsum(log_a: torch.Tensor, chunk: int, stream=None) -> torch.Tensor:
    """cs [b, H, nchunks, chunk] fp32: the within-chunk inclusive cumsum of log a."""
    b, T, H = log_a.shape
    p = make_problem(b, T, H, 16, 16, 1, chunk, 1, torch.float32)
    cs = torch.empty((b, H, -(-T // chunk), chunk), dtype=torch.float32, device=log_a.device)
    _check(lib().ssd_chunk_cumsum(ctypes.byref(p), _ptr(log_a), _ptr(cs), _stream(stream)), "ssd_chunk_cumsum")
    return cs


def chunk_state(X, B, cs, chunk, seq_idx=None, nseq=1, final_partials: Optional[torch.Tensor] = None,
                path="auto", stream=None) -> torch.Tensor:
    """Chunk end states of the last piece of each chunk (zero incoming state):
    [b, nchunks, H, N, P] fp32. Writes sequence partials into final_partials."""
    p = problem_from(X, B, chunk, nseq, path)
    b, T, H, P = X.shape
    N = B.shape[3]
    states = torch.empty((b, -(-T // chunk), H, N, P), dtype=torch.float32, device=X.device)
    _check(lib().ssd_chunk_state(ctypes.byref(p), _ptr(X), _ptr(B), _ptr(cs), _ptr(seq_idx), _ptr(states),
                                 _ptr(final_partials), _stream(stream)), "ssd_chunk_state")
    return states


def state_passing(cs, chunk_states, X_shape, dstate, ngroups, chunk, init_states=None, seq_idx=None, nseq=1,
                  final_states: Optional[torch.Tensor] = None, in_place=False, dtype=torch.bfloat16,
                  stream=None) -> torch.Tensor:
    """Incoming state of every chunk, [b, nchunks, H, N, P] fp32."""
    b, T, H, P = X_shape
    p = make_problem(b, T, H, P, dstate, ngroups, chunk, nseq, dtype)
    inc = chunk_states if in_place else torch.empty_like(chunk_states)
    _check(lib().ssd_state_passing(ctypes.byref(p), _ptr(cs), _ptr(chunk_states), _ptr(inc), _ptr(init_states),
                                   _ptr(seq_idx), _ptr(final_states), _stream(stream)), "ssd_state_passing")
    return inc


def chunk_scan(X, B, C, cs, incoming, chunk, D=None, init_states=None, seq_idx=None, nseq=1, path="auto",
               stream=None) -> torch.Tensor:
    """Y of every chunk from its incoming state (step 4)."""
    p = problem_from(X, B, chunk, nseq, path)
    Y = torch.empty_like(X)
    _check(lib().ssd_chunk_scan(ctypes.byref(p), _ptr(X), _ptr(B), _ptr(C), _ptr(cs), _ptr(D), _ptr(incoming),
                                _ptr(init_states), _ptr(seq_idx), _ptr(Y), _stream(stream)), "ssd_chunk_scan")
    return Y


# ---- the fused path, one call per kernel -------------------------------------

def fused_work_tiles(p: Problem) -> int:
    """Tiles per work range ssd_fwd uses on the fused path (-1 outside its domain)."""
    return int(lib().ssd_fused_work_tiles(ctypes.byref(p)))


def fused_work_count(p: Problem, work_tiles: int) -> int:
    """Number of work ranges for p and work_tiles (-1 if invalid)."""
    return int(lib().ssd_fused_work_count(ctypes.byref(p), int(work_tiles)))


def _fused_problem(X, B, nseq, chunk):
    return problem_from(X, B, chunk, nseq, "fused")


def segment_state(X, log_a, B, work_tiles, seq_idx=None, nseq=1, chunk=64, stream=None):
    """Right factors at the range cuts: (work_local [nwork, 2, N, P], work_decay [nwork, 2]).

    Entries of ranges that end at a row end are left as allocated (NaN here)."""
    p = _fused_problem(X, B, nseq, chunk)
    nwork = fused_work_count(p, work_tiles)
    if nwork < 0:
        raise ValueError(f"invalid work_tiles {work_tiles}")
    N, P = B.shape[3], X.shape[3]
    loc = torch.full((nwork, 2, N, P), float("nan"), dtype=torch.float32, device=X.device)
    dec = torch.full((nwork, 2), float("nan"), dtype=torch.float32, device=X.device)
    _check(lib().ssd_segment_state(ctypes.byref(p), int(work_tiles), _ptr(X), _ptr(log_a), _ptr(B), _ptr(seq_idx),
                                   _ptr(loc), _ptr(dec), _stream(stream)), "ssd_segment_state")
    return loc, dec


def segment_passing(work_local, work_decay, X, B, work_tiles, init_states=None, seq_idx=None, nseq=1, chunk=64,
                    stream=None):
    """State entering each range that starts inside a row: [nwork, 2, N, P] (NaN elsewhere)."""
    p = _fused_problem(X, B, nseq, chunk)
    inc = torch.full_like(work_local, float("nan"))
    _check(lib().ssd_segment_passing(ctypes.byref(p), int(work_tiles), _ptr(work_local), _ptr(work_decay),
                                     _ptr(init_states), _ptr(seq_idx), _ptr(inc), _stream(stream)),
           "ssd_segment_passing")
    return inc


def fused_scan(X, log_a, B, C, work_tiles, work_incoming=None, D=None, init_states=None, seq_idx=None, nseq=1,
               final_states: Optional[torch.Tensor] = None, chunk=64, stream=None) -> torch.Tensor:
    """Y from the incoming range states (and final states into final_states)."""
    p = _fused_problem(X, B, nseq, chunk)
    Y = torch.empty_like(X)
    _check(lib().ssd_fused_scan(ctypes.byref(p), int(work_tiles), _ptr(X), _ptr(log_a), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(work_incoming), _ptr(init_states), _ptr(seq_idx), _ptr(Y), _ptr(final_states),
                                _stream(stream)), "ssd_fused_scan")
    return Y


def sp_summary_workspace_bytes(p: Problem) -> int:
    n = lib().ssd_sp_summary_workspace_bytes(ctypes.byref(p))
    if n == ctypes.c_size_t(-1).value:
        _check(lib().ssd_check_problem(ctypes.byref(p)) or SSD_ERR_INVALID_ARG, "ssd_sp_summary_workspace_bytes")
    return int(n)


def sp_summary(X, log_a, B, seq_idx=None, nseq=1, chunk=64, path="auto", stream=None):
    """This rank's segment summary: (loc [b, H, N, P] fp32, dec [b, H] fp32,
    ids [b, 2] int32), with E = dec * H_start + loc over the segment's last
    sequence piece and ids its first and last sequence ids. The chunk length
    is used only where the summary runs the chunked steps (outside the fused
    family's domain)."""
    p = problem_from(X, B, chunk, nseq, path)
    b, _, H, P = X.shape
    N = B.shape[3]
    loc = torch.empty((b, H, N, P), dtype=torch.float32, device=X.device)
    dec = torch.empty((b, H), dtype=torch.float32, device=X.device)
    ids = torch.empty((b, 2), dtype=torch.int32, device=X.device)
    need = sp_summary_workspace_bytes(p)
    ws = torch.empty(need, dtype=torch.uint8, device=X.device) if need else None
    _check(lib().ssd_sp_summary(ctypes.byref(p), _ptr(X), _ptr(log_a), _ptr(B), _ptr(seq_idx), _ptr(loc), _ptr(dec),
                                _ptr(ids), _ptr(ws), need, _stream(stream)), "ssd_sp_summary")
    return loc, dec, ids


def sp_combine(X, B, g_loc, g_dec, g_ids, rank, init_states=None, nseq=1, chunk=64, stream=None):
    """Initial states [b, nseq, H, N, P] of this rank's segment from the R
    ranks' stacked summaries (g_loc [R, b, H, N, P], g_dec [R, b, H], g_ids [R, b, 2])."""
    p = problem_from(X, B, chunk, nseq)
    b, _, H, P = X.shape
    N = B.shape[3]
    init_local = torch.empty((b, nseq, H, N, P), dtype=torch.float32, device=X.device)
    _check(lib().ssd_sp_combine(ctypes.byref(p), int(g_loc.shape[0]), int(rank), _ptr(g_loc), _ptr(g_dec),
                                _ptr(g_ids), _ptr(init_states), _ptr(init_local), _stream(stream)), "ssd_sp_combine")
    return init_local


def sp_own_finals(X, B, final_states, g_ids, rank, nseq=1, chunk=64, stream=None):
    """Zero, in place, the final states of sequences this rank does not own."""
    p = problem_from(X, B, chunk, nseq)
    _check(lib().ssd_sp_own_finals(ctypes.byref(p), int(g_ids.shape[0]), int(rank), _ptr(g_ids), _ptr(final_states),
                                   _stream(stream)), "ssd_sp_own_finals")
    return final_states


def fused_scan_chained(X, log_a, B, C, work_tiles, work_local=None, work_decay=None, D=None, init_states=None,
                       seq_idx=None, nseq=1, final_states: Optional[torch.Tensor] = None, chunk=64,
                       stream=None) -> torch.Tensor:
    """Y from segment_state's range states, the cuts chained inside the scan."""
    p = _fused_problem(X, B, nseq, chunk)
    Y = torch.empty_like(X)
    _check(lib().ssd_fused_scan_chained(ctypes.byref(p), int(work_tiles), _ptr(X), _ptr(log_a), _ptr(B), _ptr(C),
                                        _ptr(D), _ptr(work_local), _ptr(work_decay), _ptr(init_states),
                                        _ptr(seq_idx), _ptr(Y), _ptr(final_states), _stream(stream)),
           "ssd_fused_scan_chained")
    return Y


def decode_step(x: torch.Tensor, log_a: torch.Tensor, B: torch.Tensor, C: torch.Tensor, state: torch.Tensor,
                D: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One step of the recurrence for every (b, h): state [b, H, N, P] fp32 is
    updated in place (state <- a state + B x^T) and y = C^T state + D x
    [b, H, P] (dtype of x) is returned. x [b, H, P], log_a [b, H] fp32,
    B and C [b, G, N]."""
    if x.dim() != 3 or B.dim() != 3 or C.shape != B.shape or log_a.shape != x.shape[:2]:
        raise ValueError("shapes: x [b,H,P], log_a [b,H], B and C [b,G,N]")
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if B.shape[0] != b or state.shape != (b, H, N, P) or state.dtype != torch.float32:
        raise ValueError("state must be float32 [b, H, N, P]")
    if x.dtype not in (torch.float32, torch.bfloat16) or B.dtype != x.dtype or C.dtype != x.dtype:
        raise TypeError("x, B and C must share one dtype, float32 or bfloat16")
    if log_a.dtype != torch.float32 or (D is not None and (D.dtype != torch.float32 or D.shape != (H,))):
        raise TypeError("log_a and D must be float32 (D [nheads])")
    p = make_problem(b, 64, H, P, N, G, 64, 1, x.dtype)  # seqlen, chunk, nseq are not read by the step
    y = torch.empty_like(x) if out is None else out
    _check(lib().ssd_decode_step(ctypes.byref(p), _ptr(x), _ptr(log_a), _ptr(B), _ptr(C), _ptr(D), _ptr(state),
                                 _ptr(y), _stream(stream)), "ssd_decode_step")
    return y


def discretize(dt: torch.Tensor, A: torch.Tensor, x: torch.Tensor, dt_bias: Optional[torch.Tensor] = None,
               zoh: bool = False, stream=None, out=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """log_a = softplus(dt + dt_bias) * A and X = s * x (s = delta, or the
    zero-order-hold (exp(delta A) - 1) / A when zoh): the log_a and X inputs of
    ssd_fwd. dt [b, T, H] fp32, A and dt_bias [H] fp32, x [b, T, H, P];
    out = (log_a, X) to write into preallocated tensors."""
    if x.dim() != 4 or dt.shape != x.shape[:3] or A.shape != (x.shape[2],):
        raise ValueError("shapes: x [b,T,H,P], dt [b,T,H], A [H]")
    if dt.dtype != torch.float32 or A.dtype != torch.float32 or (dt_bias is not None and dt_bias.dtype != torch.float32):
        raise TypeError("dt, A and dt_bias must be float32")
    b, T, H, P = x.shape
    p = make_problem(b, T, H, P, 16, 1, 64, 1, x.dtype)  # dstate, ngroups, chunk are not read by this step
    if out is None:
        log_a = torch.empty(dt.shape, dtype=torch.float32, device=dt.device)
        X = torch.empty_like(x)
    else:
        log_a, X = out
    _check(lib().ssd_discretize(ctypes.byref(p), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(x), int(bool(zoh)),
                                _ptr(log_a), _ptr(X), _stream(stream)), "ssd_discretize")
    return log_a, X
