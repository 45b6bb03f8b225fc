"""Randomised parity: problems drawn from a fixed seed over the shapes the
library accepts (ragged T, every supported P and N, grouped B/C, both dtypes,
packed sequences including ids that never occur, D and initial states on or
off), each run through every family that covers it and compared with the CPU
fp64 oracle under the parity rule max|gpu - oracle| <= tau * max|oracle|
(tau = 1e-5 for fp32 inputs, 2e-2 for bf16 inputs with fp32 state).
"""
import os

import numpy as np
import pytest
import torch

from gpu_util import TAU, assert_close, run_gpu, run_oracle
from workloads import make_custom

pytestmark = pytest.mark.gpu

# more problems for a longer stress run: SSD_RANDOM_PROBLEMS=400 pytest ...
NPROBLEMS = int(os.environ.get("SSD_RANDOM_PROBLEMS", "64"))


def _draw(i):
    """Problem i: (inputs, dtype, chunk, description)."""
    rng = np.random.default_rng(7000 + i)
    dtype = "bf16" if rng.random() < 0.6 else "f32"
    b = int(rng.integers(1, 3))
    T = int(rng.integers(1, 700))
    P = int(rng.choice([16, 32, 64, 64]))
    N = int(rng.choice([16, 32, 48, 64, 128, 128, 256]))
    H = int(rng.integers(1, 9))
    G = int(rng.choice([g for g in range(1, H + 1) if H % g == 0]))
    Q = int(rng.choice([64, 128, 256]))
    lengths = None
    if rng.random() < 0.6:
        lengths = []
        nseq = int(rng.integers(1, 6))
        for _ in range(b):
            cuts = np.sort(rng.integers(0, T + 1, size=nseq - 1))
            parts = np.diff(np.concatenate([[0], cuts, [T]])).astype(int).tolist()
            lengths.append(parts)
    D = str(rng.choice(["none", "normal", "ones"]))
    init = bool(rng.random() < 0.5)
    nseq = None if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, ngroups=G, dtype=dtype, seed=int(rng.integers(0, 10000)), has_D=D,
                    has_init=init, lengths=lengths, nseq=nseq)
    desc = f"{dtype} b{b} T{T} H{H} G{G} P{P} N{N} Q{Q} seqs={lengths} D={D} init={init}"
    return d, dtype, Q, desc


@pytest.mark.parametrize("i", range(NPROBLEMS))
def test_random_problem_every_family(i):
    import mamba_ssd_layer_chunked_b200 as ssd
    d, dtype, Q, desc = _draw(i)
    Yr, Fr = run_oracle(d)
    X = d["X"]
    p = ssd.make_problem(X.shape[0], X.shape[1], X.shape[2], X.shape[3], d["B"].shape[3], d["B"].shape[2], Q,
                         d["nseq"], torch.bfloat16 if dtype == "bf16" else torch.float32)
    ran = 0
    for path in ("auto", "simt", "fused"):
        if path != "auto" and not ssd.path_supported(p, path):
            continue
        Y, F = run_gpu(d, dtype, Q, path)
        assert_close(Y, Yr, TAU[dtype], f"Y ({path}; {desc})")
        assert_close(F, Fr, TAU[dtype], f"final_states ({path}; {desc})")
        ran += 1
    assert ran >= 2  # auto and at least the SIMT family


NLARGE = 8


def _draw_large(i):
    """Larger bf16 problems in the fused family's domain, long enough that its
    work ranges cut rows and chain the pieces before each cut."""
    rng = np.random.default_rng(9000 + i)
    b = int(rng.integers(1, 4))
    T = int(rng.integers(1000, 4097))
    H = int(rng.choice([2, 4, 6, 8]))
    G = int(rng.choice([g for g in (1, 2) if (H // g) % 2 == 0 and H % g == 0]))
    N = int(rng.choice([64, 128]))
    Q = int(rng.choice([128, 256]))
    lengths = None
    if rng.random() < 0.5:
        nseq = int(rng.integers(1, 9))
        lengths = []
        for _ in range(b):
            cuts = np.sort(rng.integers(0, T + 1, size=nseq - 1))
            lengths.append(np.diff(np.concatenate([[0], cuts, [T]])).astype(int).tolist())
    D = str(rng.choice(["none", "normal"]))
    init = bool(rng.random() < 0.5)
    nseq = None if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, 64, N, ngroups=G, dtype="bf16", seed=int(rng.integers(0, 10000)), has_D=D,
                    has_init=init, lengths=lengths, nseq=nseq)
    return d, Q, f"bf16 b{b} T{T} H{H} G{G} N{N} Q{Q} nseq={nseq} D={D} init={init}"


@pytest.mark.parametrize("i", range(NLARGE))
def test_random_large_problem_fused_and_chunked(i):
    import mamba_ssd_layer_chunked_b200 as ssd
    d, Q, desc = _draw_large(i)
    Yr, Fr = run_oracle(d)
    X = d["X"]
    p = ssd.make_problem(X.shape[0], X.shape[1], X.shape[2], 64, d["B"].shape[3], d["B"].shape[2], Q, d["nseq"],
                         torch.bfloat16)
    assert ssd.path_supported(p, "fused")
    for path in ("auto", "fused"):
        if not ssd.path_supported(p, path) and path != "auto":
            continue
        Y, F = run_gpu(d, "bf16", Q, path)
        assert_close(Y, Yr, TAU["bf16"], f"Y ({path}; {desc})")
        assert_close(F, Fr, TAU["bf16"], f"final_states ({path}; {desc})")


NWIDE = 16


def _draw_wide(i):
    """Problems that the fused family runs as 64-column slots other than a plain
    head pair: head dimension 128 (one head per row), or an odd number of heads
    per group (the last pair of each group half empty). Long enough, for some,
    that the work ranges cut rows."""
    rng = np.random.default_rng(11000 + i)
    b = int(rng.integers(1, 3))
    T = int(rng.choice([int(rng.integers(1, 600)), int(rng.integers(1500, 3500))]))
    if i % 2 == 0:
        P, H = 128, int(rng.integers(1, 5))
        G = int(rng.choice([g for g in range(1, H + 1) if H % g == 0]))
    else:
        P = 64
        G = int(rng.integers(1, 3))
        H = G * int(rng.choice([1, 3, 5]))
    N = int(rng.choice([32, 64, 128, 128, 256]))
    Q = int(rng.choice([64, 128, 256]))
    lengths = None
    if rng.random() < 0.6:
        nseq = int(rng.integers(1, 6))
        lengths = []
        for _ in range(b):
            cuts = np.sort(rng.integers(0, T + 1, size=nseq - 1))
            lengths.append(np.diff(np.concatenate([[0], cuts, [T]])).astype(int).tolist())
    D = str(rng.choice(["none", "normal"]))
    init = bool(rng.random() < 0.5)
    nseq = None if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, ngroups=G, dtype="bf16", seed=int(rng.integers(0, 10000)), has_D=D,
                    has_init=init, lengths=lengths, nseq=nseq)
    return d, Q, f"bf16 b{b} T{T} H{H} G{G} P{P} N{N} Q{Q} nseq={nseq} D={D} init={init}"


@pytest.mark.parametrize("i", range(NWIDE))
def test_random_wide_slots_fused(i):
    import mamba_ssd_layer_chunked_b200 as ssd
    d, Q, desc = _draw_wide(i)
    X = d["X"]
    p = ssd.make_problem(X.shape[0], X.shape[1], X.shape[2], X.shape[3], d["B"].shape[3], d["B"].shape[2], Q,
                         d["nseq"], torch.bfloat16)
    assert ssd.path_supported(p, "fused"), desc
    Yr, Fr = run_oracle(d)
    for path in ("auto", "fused"):
        Y, F = run_gpu(d, "bf16", Q, path)
        assert_close(Y, Yr, TAU["bf16"], f"Y ({path}; {desc})")
        assert_close(F, Fr, TAU["bf16"], f"final_states ({path}; {desc})")
