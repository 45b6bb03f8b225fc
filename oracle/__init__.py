"""CPU fp64 oracle for the SSD chunked-scan forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` are the only users. The product path
(the C-ABI library and its Python binding) never imports this package, and
this package imports nothing from the product.

Contents
--------
``ssd_reference``      the step-by-step fp64 recurrence (plain C, OpenMP over
                       batch x heads), the oracle every parity test compares to.
``chunk_states``       states at chunk boundaries from the same recurrence, to
                       localise errors in the chunked path.
``chunk_cumsum``       the within-chunk inclusive cumulative sum of log a (a
                       NumPy one-liner: the definition of the quantity).
``segment_decay``      the product of a over each chunk's last sequence piece.
``dual_matrix``        brute-force matrix form M = L * (C B^T) (+ init and D
                       terms), Y = M X, in NumPy fp64, tiny sizes only.
``blockwise``          the pages' four-step block algorithm in NumPy fp64
                       (diagonal blocks, chunk end states, state scan, incoming
                       output), tiny sizes only.
``recurrence_numpy``   a NumPy twin of the C recurrence for tiny inputs (used to
                       show that the pins catch planted mistakes).
``discretize``         the step before the scan: softplus step size, log a = delta A,
                       and x scaled by delta (or by the zero-order hold factor).

Every function takes and returns NumPy arrays; floating inputs are read as
float64 (bf16/fp32 input values convert exactly).
"""
from .ssd_oracle import (  # noqa: F401
    ssd_reference,
    chunk_states,
    chunk_cumsum,
    segment_decay,
    dual_matrix,
    blockwise,
    recurrence_numpy,
    discretize,
    oracle_library_path,
    build_oracle,
    max_threads,
)
