"""fp64 oracle functions for the SSD forward (test infrastructure only).

Sources, by page title and section:

* "Mamba-2: writing the recurrent state as a structured matrix"
  (wq-win.github.io/llm/088-mamba2.html), section 2.1 (the recurrence
  H_t = a_t H_{t-1} + B_t x_t^T, y_t = C_t^T H_t, and its unrolled sum with the
  empty product equal to 1), section 2.2 (the lower-triangular L with
  L_ts = prod_{j=s+1..t} a_j and the dual form Y = [L o (C B^T)] X), section 2.3
  (chunks of length Q: a local output with zero incoming state plus the
  contribution of the state carried in), section 3 (the block algorithm:
  per-chunk L, local output, local end state, block decay; a scan over chunks;
  the incoming state decayed to each position and read out by C), and the
  worked examples of sections 2.2-2.3.
* "Mamba-2 - Transformer and SSM share one algebra" (awesome.papernotes.org,
  2024_mamba2), design 2 "SSD algorithm" (the chunked cumulative sum of the
  decays and L = exp(segment sum)).
* "Mamba and state space models" (wang-x-xia.github.io learn-ai foundations),
  section 2 (discrete form y_t = C h_t + D x_t).

Conventions shared by every function here (and stated in the C file):
init_states is the state before the first token (H_{-1}); a change of seq_idx
starts an independent sequence from its own initial state (or zero); head h uses
group h // (nheads // ngroups); D is a per-head scalar on the skip path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None


def oracle_library_path() -> str:
    return _LIB


def build_oracle(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, OpenMP) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_oracle())
            i64, dp, ip = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int32)
            lib.ssd_oracle_fwd.argtypes = [i64] * 7 + [dp] * 6 + [ip, dp, dp, ctypes.c_int]
            lib.ssd_oracle_fwd.restype = ctypes.c_int
            lib.ssd_oracle_chunk_states.argtypes = [i64] * 8 + [dp] * 4 + [ip, dp, dp, ctypes.c_int]
            lib.ssd_oracle_chunk_states.restype = ctypes.c_int
            lib.ssd_oracle_max_threads.argtypes = []
            lib.ssd_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().ssd_oracle_max_threads())


def _f64(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _dims(X, B, seq_idx, nseq):
    batch, seqlen, nheads, headdim = X.shape
    _, _, ngroups, dstate = B.shape
    if nseq is None:
        nseq = 1 if seq_idx is None else int(np.max(seq_idx)) + 1 if seq_idx.size else 1
    return batch, seqlen, nheads, headdim, dstate, ngroups, nseq


def ssd_reference(X, log_a, B, C, D=None, init_states=None, seq_idx=None, nseq=None,
                  nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Step-by-step fp64 recurrence. Returns (Y, final_states)."""
    X, log_a, B, C, D, init = (_f64(v) for v in (X, log_a, B, C, D, init_states))
    si = None if seq_idx is None else np.ascontiguousarray(np.asarray(seq_idx, dtype=np.int32))
    batch, seqlen, nheads, headdim, dstate, ngroups, ns = _dims(X, B, si, nseq)
    Y = np.empty_like(X)
    final = np.empty((batch, ns, nheads, dstate, headdim), dtype=np.float64)
    rc = _load().ssd_oracle_fwd(batch, seqlen, nheads, headdim, dstate, ngroups, ns,
                                _ptr(X), _ptr(log_a), _ptr(B), _ptr(C), _ptr(D), _ptr(init),
                                _ptr(si, ctypes.c_int32), _ptr(Y), _ptr(final), int(nthreads))
    if rc != 0:
        raise ValueError(f"ssd_oracle_fwd failed with code {rc}")
    return Y, final


def chunk_states(X, log_a, B, chunk, init_states=None, seq_idx=None, nseq=None,
                 nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """(incoming, local) states per chunk, [batch, nchunks, nheads, dstate, headdim].

    incoming: the state just before each chunk's first token for that token's
    sequence. local: the end-of-chunk state of the chunk's last sequence piece
    started from zero (the per-chunk "right factor" of the block algorithm).
    """
    X, log_a, B, init = (_f64(v) for v in (X, log_a, B, init_states))
    si = None if seq_idx is None else np.ascontiguousarray(np.asarray(seq_idx, dtype=np.int32))
    batch, seqlen, nheads, headdim, dstate, ngroups, ns = _dims(X, B, si, nseq)
    nchunks = (seqlen + chunk - 1) // chunk  # the last chunk may be shorter
    inc = np.empty((batch, nchunks, nheads, dstate, headdim), dtype=np.float64)
    loc = np.empty_like(inc)
    rc = _load().ssd_oracle_chunk_states(batch, seqlen, nheads, headdim, dstate, ngroups, ns, chunk,
                                         _ptr(X), _ptr(log_a), _ptr(B), _ptr(init),
                                         _ptr(si, ctypes.c_int32), _ptr(inc), _ptr(loc), int(nthreads))
    if rc != 0:
        raise ValueError(f"ssd_oracle_chunk_states failed with code {rc}")
    return inc, loc


def chunk_cumsum(log_a, chunk) -> np.ndarray:
    """Inclusive cumulative sum of log a within each chunk: [batch, nheads, nchunks, chunk].

    cs[b, h, c, k] = sum_{j <= k} log_a[b, c*chunk + j, h] (papernotes design 2:
    A_cumsum over the within-chunk axis).
    """
    la = np.asarray(log_a, dtype=np.float64)
    batch, seqlen, nheads = la.shape
    nchunks = seqlen // chunk
    la = la.reshape(batch, nchunks, chunk, nheads).transpose(0, 3, 1, 2)
    return np.cumsum(la, axis=-1)


def segment_decay(log_a, chunk, seq_idx=None) -> np.ndarray:
    """Product of a_t over the last sequence piece of each chunk (the block decay
    of wq-win 088 section 3 for a block that may hold a sequence start):
    [batch, nchunks, nheads], nchunks = ceil(seqlen / chunk)."""
    la = np.asarray(log_a, dtype=np.float64)
    batch, seqlen, nheads = la.shape
    nch = (seqlen + chunk - 1) // chunk
    seq = np.zeros((batch, seqlen), dtype=np.int64) if seq_idx is None else np.asarray(seq_idx, np.int64)
    out = np.zeros((batch, nch, nheads))
    for b in range(batch):
        for c in range(nch):
            t1 = min(seqlen, (c + 1) * chunk)
            st = t1 - 1
            while st > c * chunk and seq[b, st - 1] == seq[b, t1 - 1]:
                st -= 1
            out[b, c] = np.exp(la[b, st:t1].sum(axis=0))
    return out


def _group_of(h, nheads, ngroups):
    return h // (nheads // ngroups)


def dual_matrix(X, log_a, B, C, D=None, init_states=None, seq_idx=None, nseq=None,
                return_M: bool = False):
    """Brute-force matrix ("dual") form, fp64, O(T^2) per head.

    For each (b, h): M[t, s] = L[t, s] * (C_t . B_s) with
    L[t, s] = prod_{j=s+1..t} a_j for s <= t in the same sequence, else 0
    (wq-win 088, section 2.2). The initial state of the sequence of token t,
    started at token st, contributes (prod_{j=st..t} a_j) C_t^T H0 (the unrolled
    sum with a non-zero H_{-1}). Y = M X + D x. Returns Y (and M if asked,
    [batch, nheads, T, T]).
    """
    X, la, B, C = (np.asarray(v, dtype=np.float64) for v in (X, log_a, B, C))
    batch, seqlen, nheads, headdim = X.shape
    ngroups = B.shape[2]
    seq = np.zeros((batch, seqlen), dtype=np.int64) if seq_idx is None else np.asarray(seq_idx, np.int64)
    Y = np.zeros_like(X)
    Ms = np.zeros((batch, nheads, seqlen, seqlen)) if return_M else None
    t_idx = np.arange(seqlen)
    for b in range(batch):
        same = seq[b][:, None] == seq[b][None, :]
        causal = t_idx[:, None] >= t_idx[None, :]
        for h in range(nheads):
            g = _group_of(h, nheads, ngroups)
            a = np.exp(la[b, :, h])
            # L[t, s] = prod_{j=s+1..t} a_j, built by explicit products
            L = np.zeros((seqlen, seqlen))
            for t in range(seqlen):
                prod = 1.0
                L[t, t] = 1.0
                for s in range(t - 1, -1, -1):
                    prod *= a[s + 1]
                    L[t, s] = prod
            L = np.where(causal & same, L, 0.0)
            M = L * (C[b, :, g, :] @ B[b, :, g, :].T)
            y = M @ X[b, :, h, :]
            if init_states is not None:
                H0 = np.asarray(init_states, dtype=np.float64)
                for t in range(seqlen):
                    st = t
                    while st > 0 and seq[b, st - 1] == seq[b, t]:
                        st -= 1
                    decay = np.prod(a[st:t + 1])
                    y[t] += decay * (C[b, t, g, :] @ H0[b, seq[b, t], h])
            if D is not None:
                y += np.asarray(D, dtype=np.float64)[h] * X[b, :, h, :]
            Y[b, :, h, :] = y
            if return_M:
                Ms[b, h] = M
    return (Y, Ms) if return_M else Y


def blockwise(X, log_a, B, C, chunk, D=None, init_states=None, return_parts: bool = False):
    """The pages' block algorithm in fp64 for one sequence per batch row.

    wq-win 088 section 3 / papernotes design 2, in their order:
      1. per chunk: L = exp(segment sum of log a); local output (L o C B^T) X
         with zero incoming state; local end state sum_s (prod_{j>s} a_j) B_s x_s^T;
         block decay = product of the chunk's a_t.
      2. scan over chunks: real_end = block_decay * previous + local_end,
         starting from the initial state (zero if None).
      3. per chunk: the incoming state decayed to each position and read out by C,
         added to the local output.
    Returns Y [+ D x] and, when return_parts, a dict with the per-chunk pieces
    (local_out, incoming_out, local_end, block_decay, incoming_state, final).
    """
    X, la, B, C = (np.asarray(v, dtype=np.float64) for v in (X, log_a, B, C))
    batch, seqlen, nheads, headdim = X.shape
    ngroups, dstate = B.shape[2], B.shape[3]
    if seqlen % chunk:
        raise ValueError("seqlen must be a multiple of chunk")
    nch = seqlen // chunk
    Y = np.zeros_like(X)
    parts = dict(local_out=np.zeros((batch, nheads, nch, chunk, headdim)),
                 incoming_out=np.zeros((batch, nheads, nch, chunk, headdim)),
                 local_end=np.zeros((batch, nheads, nch, dstate, headdim)),
                 block_decay=np.zeros((batch, nheads, nch)),
                 incoming_state=np.zeros((batch, nheads, nch, dstate, headdim)),
                 final=np.zeros((batch, nheads, dstate, headdim)))
    for b in range(batch):
        for h in range(nheads):
            g = _group_of(h, nheads, ngroups)
            local_out, local_end, block_decay, cums = [], [], [], []
            for c in range(nch):
                sl = slice(c * chunk, (c + 1) * chunk)
                cs = np.cumsum(la[b, sl, h])  # within-chunk cumulative sum
                seg = cs[:, None] - cs[None, :]  # segment sum over (s, t]
                lower = np.tril(np.ones((chunk, chunk), dtype=bool))
                Lc = np.exp(np.where(lower, seg, -np.inf))  # exp(segment sum), 0 above the diagonal
                Cc, Bc, Xc = C[b, sl, g, :], B[b, sl, g, :], X[b, sl, h, :]
                local_out.append((Lc * (Cc @ Bc.T)) @ Xc)
                decay_to_end = np.exp(cs[-1] - cs)  # prod_{j=s+1..end} a_j
                local_end.append(Bc.T @ (decay_to_end[:, None] * Xc))
                block_decay.append(np.exp(cs[-1]))
                cums.append(cs)
            state = (np.zeros((dstate, headdim)) if init_states is None
                     else np.asarray(init_states, dtype=np.float64)[b, 0, h].copy())
            for c in range(nch):
                sl = slice(c * chunk, (c + 1) * chunk)
                parts["incoming_state"][b, h, c] = state
                inc_out = np.exp(cums[c])[:, None] * (C[b, sl, g, :] @ state)
                Y[b, sl, h, :] = local_out[c] + inc_out
                parts["local_out"][b, h, c] = local_out[c]
                parts["incoming_out"][b, h, c] = inc_out
                parts["local_end"][b, h, c] = local_end[c]
                parts["block_decay"][b, h, c] = block_decay[c]
                state = block_decay[c] * state + local_end[c]
            parts["final"][b, h] = state
            if D is not None:
                Y[b, :, h, :] += np.asarray(D, dtype=np.float64)[h] * X[b, :, h, :]
    return (Y, parts) if return_parts else Y


def recurrence_numpy(X, log_a, B, C, D=None, init_states=None, seq_idx=None, nseq=None,
                     _mutation: Optional[str] = None):
    """NumPy twin of the C recurrence (tiny inputs). ``_mutation`` plants a
    deliberate mistake for the test that checks the pins catch it; it is never
    set outside that test."""
    X, la, B, C = (np.asarray(v, dtype=np.float64) for v in (X, log_a, B, C))
    batch, seqlen, nheads, headdim = X.shape
    ngroups, dstate = B.shape[2], B.shape[3]
    seq = np.zeros((batch, seqlen), dtype=np.int64) if seq_idx is None else np.asarray(seq_idx, np.int64)
    ns = (int(seq.max()) + 1 if seqlen else 1) if nseq is None else nseq
    init = None if init_states is None else np.asarray(init_states, dtype=np.float64)
    Y = np.zeros_like(X)
    final = np.zeros((batch, ns, nheads, dstate, headdim))
    m = _mutation
    for b in range(batch):
        for h in range(nheads):
            g = _group_of(h, nheads, ngroups)
            if init is not None:
                final[b, :, h] = init[b, :, h]
            cur = seq[b, 0] if seqlen else 0
            H = np.zeros((dstate, headdim)) if init is None else init[b, cur, h].copy()
            for t in range(seqlen):
                s = seq[b, t]
                if t > 0 and s != cur and m != "no_reset":
                    final[b, cur, h] = H
                    cur = s
                    H = np.zeros((dstate, headdim)) if init is None else init[b, cur, h].copy()
                if m == "decay_index" and t > 0:
                    a = np.exp(la[b, t - 1, h])
                elif m == "decay_sign":
                    a = np.exp(-la[b, t, h])
                else:
                    a = np.exp(la[b, t, h])
                w, r = (C, B) if m == "swap_BC" else (B, C)
                if m == "undecayed_init" and t == 0:
                    a = 1.0
                H = a * H + np.outer(w[b, t, g, :], X[b, t, h, :])
                y = r[b, t, g, :] @ H
                if D is not None and m != "drop_D":
                    y = y + np.asarray(D, dtype=np.float64)[h] * X[b, t, h, :]
                if m == "transpose_readout" and dstate == headdim:
                    y = H @ r[b, t, g, :]
                Y[b, t, h, :] = y
            if seqlen:
                final[b, cur, h] = H
    return Y, final


def discretize(dt, A, x, dt_bias=None, zoh: bool = False):
    """The step before the scan in the Mamba block, fp64: (log_a [b,T,H], X [b,T,H,P]).

    delta = softplus(dt + dt_bias) and A_bar = exp(delta A) (the Mamba page,
    ai.tomabc.com paper story 21: the block pseudocode and the discretisation of
    A); B_bar x is delta B x (zoh False) or the zero-order hold
    (exp(delta A) - 1) / A B x ("Mamba and state space models", section 2), the
    scalar put on x: log_a = delta A, X = s x.
    """
    dt = np.asarray(dt, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    z = dt + (0.0 if dt_bias is None else np.asarray(dt_bias, dtype=np.float64))
    delta = np.logaddexp(0.0, z)  # log(1 + e^z)
    log_a = delta * A
    if zoh:
        nz = A != 0.0
        s = np.where(nz, np.expm1(log_a) / np.where(nz, A, 1.0), delta)
    else:
        s = delta
    X = s[..., None] * np.asarray(x, dtype=np.float64)
    return log_a, X
