"""B200 (sm_100a) SSD chunked-scan forward: a C-ABI CUDA library
(libssd_b200.so, include/ssd.h) and its thin Python binding.

    from mamba_ssd_layer_chunked_b200 import ssd_fwd
    Y, final_states = ssd_fwd(X, log_a, B, C, chunk=256, D=D, init_states=h0,
                              seq_idx=seq_idx, nseq=nseq)

Importing the package loads the library and raises ImportError when it has
not been built (``python mamba_ssd_layer_chunked_b200/build.py``): there is no
fallback implementation.
"""
from .ssd import (  # noqa: F401
    LIB_PATH,
    Problem,
    SSDError,
    chunk_cumsum,
    chunk_scan,
    chunk_state,
    decode_step,
    discretize,
    check_device_error,
    declared_functions,
    device_error,
    fused_scan,
    fused_scan_chained,
    fused_work_count,
    fused_work_tiles,
    segment_passing,
    segment_state,
    selftest_wait_timeout,
    sp_combine,
    sp_own_finals,
    sp_summary,
    lib,
    make_problem,
    path_supported,
    problem_from,
    ssd_fwd,
    ssd_fwd_host,
    state_passing,
    states_bytes,
    status_string,
    workspace_bytes,
)

from .sp import ssd_fwd_sp, torch_collectives  # noqa: F401,E402

lib()  # fail loudly at import when the CUDA library is missing
