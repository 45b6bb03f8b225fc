"""Seeded synthetic inputs for the SSD chunked-scan forward.

This module is shared by the CPU oracle tests, the GPU parity tests and
``bench.py``. It draws random inputs and nothing else: it holds none of the
method's arithmetic (no decay products, no state updates, no matrix forms).

The workloads follow the shapes and value distributions the Mamba-2 pages use
for the SSD layer (scalar decay per head, head dim P, state dim N, B and C
shared across the heads of a group, packed variable-length batches with
per-sequence initial states):

* X ~ N(0, 1); B, C ~ N(0, 1/N).
* Tiny fp32 case: log a = -Delta with Delta ~ U[0.01, 0.5] per (b, t, h).
* Mamba-2-shaped layers: Delta = softplus(z), z ~ N(-3, 1) per (b, t, h);
  A_log ~ U[0, ln 16] per head; log a = -Delta * exp(A_log). This is the
  standard zero-order-hold parameterisation a = exp(Delta * A) with A < 0, drawn
  here only to give log a the distribution of a trained layer.
* bf16 workloads round X, B and C to bfloat16 (round to nearest even) before
  anything else sees them, so the oracle and the GPU read identical values.
  log a, D and the initial states stay fp32.

Every array is a NumPy array. bf16 values are returned as float32 arrays whose
values are exactly representable in bfloat16.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "round_to_bf16",
    "make_inputs",
    "make_custom",
    "varlen_lengths",
    "seq_idx_from_lengths",
]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); return float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return rounded.view(np.float32).reshape(x.shape)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and value recipe."""

    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int  # P
    dstate: int  # N
    ngroups: int  # G
    chunk: int  # Q
    dtype: str  # "f32" or "bf16": dtype of X, B, C and Y
    seed: int
    decay: str  # "uniform" (tiny case) or "softplus" (Mamba-2-shaped layers)
    has_D: str  # "none", "ones" or "normal"
    has_init: bool
    nseq: int = 1  # sequences per batch row
    varlen: str = "none"  # "none", "half" (reset at T/2) or "packed"

    @property
    def tokens_heads(self) -> int:
        return self.batch * self.seqlen * self.nheads


# The five workloads of the Mamba-2 SSD layer study (tiny parity case, the
# 130M- and 2.7B-shaped layers, the long-sequence state-size sweep and the packed
# variable-length batch). Seeds: 1000 + k, and 1040 + N for the N sweep.
WORKLOADS: Dict[str, Workload] = {}


def _add(w: Workload) -> None:
    WORKLOADS[w.name] = w


_add(Workload("tiny_f32", 1, 256, 2, 16, 16, 1, 64, "f32", 1001, "uniform", "ones", False, 2, "half"))
_add(Workload("mamba2_130m_layer", 8, 2048, 24, 64, 128, 1, 256, "bf16", 1002, "softplus", "none", False))
_add(Workload("mamba2_2p7b_layer", 4, 4096, 80, 64, 128, 1, 256, "bf16", 1003, "softplus", "normal", False))
for _n in (16, 64, 128, 256):
    _add(Workload(f"long16k_N{_n}", 1, 16384, 80, 64, _n, 1, 256, "bf16", 1040 + _n, "softplus", "none", True))
_add(Workload("packed_varlen", 1, 32768, 24, 64, 128, 1, 256, "bf16", 1005, "softplus", "none", True, 16, "packed"))


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def varlen_lengths(rng: np.random.Generator, total: int, nseq: int,
                   lo: float = 256.0, hi: float = 4096.0) -> np.ndarray:
    """Sequence lengths drawn U[lo, hi], scaled to sum to ``total``.

    floor(u * total / sum(u)), then +1 on the first (total - sum) sequences.
    """
    u = rng.uniform(lo, hi, nseq)
    lens = np.floor(u * total / u.sum()).astype(np.int64)
    short = total - int(lens.sum())
    lens[:short] += 1
    assert int(lens.sum()) == total and (lens > 0).all()
    return lens


def seq_idx_from_lengths(lengths: Sequence[int]) -> np.ndarray:
    """Sequence index per token for consecutive sequences of the given lengths."""
    return np.repeat(np.arange(len(lengths), dtype=np.int32), np.asarray(lengths, dtype=np.int64))


def _draw(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def make_custom(batch: int, seqlen: int, nheads: int, headdim: int, dstate: int,
                ngroups: int = 1, dtype: str = "bf16", seed: int = 0,
                decay: str = "softplus", has_D: str = "none", has_init: bool = False,
                lengths: Optional[Sequence[Sequence[int]]] = None,
                nseq: Optional[int] = None) -> Dict[str, object]:
    """Draw one input set.

    ``lengths``: per batch row, the lengths of its consecutive sequences (they
    must sum to ``seqlen``); None means one sequence per row and no seq_idx.
    Returns a dict with X, log_a, B, C, D, init_states, seq_idx, nseq.
    Draw order is fixed: X, B, C, decay parameters, D, initial states.
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError(dtype)
    rng = np.random.default_rng(seed)
    X = _draw(rng, (batch, seqlen, nheads, headdim))
    B = _draw(rng, (batch, seqlen, ngroups, dstate), 1.0 / np.sqrt(dstate))
    C = _draw(rng, (batch, seqlen, ngroups, dstate), 1.0 / np.sqrt(dstate))
    if decay == "uniform":
        delta = rng.uniform(0.01, 0.5, (batch, seqlen, nheads)).astype(np.float32)
        log_a = (-delta).astype(np.float32)
    elif decay == "softplus":
        a_log = rng.uniform(0.0, np.log(16.0), nheads)
        z = rng.normal(-3.0, 1.0, (batch, seqlen, nheads))
        delta = np.log1p(np.exp(z))
        log_a = (-delta * np.exp(a_log)[None, None, :]).astype(np.float32)
    else:
        raise ValueError(decay)
    if has_D == "none":
        D = None
    elif has_D == "ones":
        D = np.ones(nheads, dtype=np.float32)
    elif has_D == "normal":
        D = rng.standard_normal(nheads, dtype=np.float32)
    else:
        raise ValueError(has_D)
    if lengths is None:
        seq_idx = None
        ns = 1 if nseq is None else nseq
    else:
        rows = [seq_idx_from_lengths(l) for l in lengths]
        if len(rows) != batch or any(r.shape[0] != seqlen for r in rows):
            raise ValueError("lengths must give seqlen tokens for each batch row")
        seq_idx = np.stack(rows).astype(np.int32)
        ns = int(seq_idx.max()) + 1 if nseq is None else nseq
    init = _draw(rng, (batch, ns, nheads, dstate, headdim)) if has_init else None
    if dtype == "bf16":
        X, B, C = round_to_bf16(X), round_to_bf16(B), round_to_bf16(C)
    return dict(X=X, log_a=log_a, B=B, C=C, D=D, init_states=init, seq_idx=seq_idx, nseq=ns)


def make_inputs(w: Workload) -> Dict[str, object]:
    """Inputs of a named workload (see ``WORKLOADS``)."""
    lengths = None
    if w.varlen == "half":
        lengths = [[w.seqlen // 2, w.seqlen - w.seqlen // 2]] * w.batch
    elif w.varlen == "packed":
        rng = np.random.default_rng(w.seed + 7919)
        lengths = [list(varlen_lengths(rng, w.seqlen, w.nseq)) for _ in range(w.batch)]
    return make_custom(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                       w.dtype, w.seed, w.decay, w.has_D, w.has_init, lengths,
                       nseq=(w.nseq if lengths is not None else None))
