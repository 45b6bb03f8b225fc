"""Sequence parallelism on one GPU: R ranks emulated as threads of one
process, each holding consecutive token segments of every batch row and
exchanging its segment summary through in-process collectives. The assembled
Y and the final states are compared with the fp64 oracle run on the whole
sequence, under the parity rule max|got - ref| <= tau * max|ref| (tau = 2e-2
for bf16 inputs with fp32 state). The segment summaries themselves are
compared with the oracle's state after the segment's last sequence piece.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TAU, assert_close, run_oracle, to_device
from workloads import make_custom

pytestmark = pytest.mark.gpu

# name: (batch, T, H, N, segment lengths, sequence lengths per row, D, init)
CASES = {
    "two_equal_one_sequence": (2, 1024, 4, 128, [512, 512], None, "none", True),
    "three_ragged_segments": (2, 1000, 4, 128, [256, 384, 360], None, "normal", True),
    "four_segments_N64_zero_init": (1, 1024, 4, 64, [256, 256, 256, 256], None, "none", False),
    # a sequence boundary exactly at the first segment boundary, others inside
    "varlen_boundary_at_segment_edge": (2, 1024, 4, 128, [256, 384, 384], [[100, 156, 400, 368], [1024]],
                                        "normal", True),
    # ids that never occur, one sequence over three segments, one starting at a rank
    "skipped_ids": (2, 768, 4, 128, [256, 256, 256], [[100, 0, 412, 0, 256], [0, 768, 0, 0, 0]], "normal", True),
    # one short segment holding only the middle of a sequence
    "short_middle_segment": (1, 640, 2, 128, [300, 40, 300], [[200, 400, 40]], "none", True),
}
# outside segment_state's domain the summary runs the chunked steps:
# name: (batch, T, H, P, N, segments, lengths, D, init, dtype, chunk)
GENERAL = {
    "f32_tiny_shape_reset": (1, 256, 2, 16, 16, [100, 156], [[128, 128]], "normal", True, "f32", 64),
    "bf16_N16": (1, 1024, 4, 64, 16, [512, 512], None, "normal", True, "bf16", 256),
    "bf16_N256_varlen": (1, 1024, 4, 64, 256, [300, 724], [[600, 424]], "normal", True, "bf16", 256),
    "bf16_P32_three_ranks": (2, 768, 4, 32, 128, [200, 300, 268], None, "none", True, "bf16", 128),
}


def _ssd():
    import mamba_ssd_layer_chunked_b200 as ssd
    return ssd


class ThreadGroup:
    """all_gather / all_reduce_sum among R threads of one process."""

    def __init__(self, nranks):
        self.nranks = nranks
        self.barrier = threading.Barrier(nranks, timeout=60)
        self.slots = [None] * nranks

    def _exchange(self, rank, t):
        self.slots[rank] = t
        self.barrier.wait()
        parts = list(self.slots)
        self.barrier.wait()
        return parts

    def collectives(self, rank):
        def all_gather(t):
            return torch.stack(self._exchange(rank, t))

        def all_reduce_sum(t):
            return torch.stack(self._exchange(rank, t)).sum(dim=0)

        return all_gather, all_reduce_sum


def _segments(g, seg):
    bounds = np.cumsum([0] + list(seg))
    out = []
    for r in range(len(seg)):
        a, b = int(bounds[r]), int(bounds[r + 1])
        out.append({k: (None if g[k] is None else g[k][:, a:b].contiguous())
                    for k in ("X", "log_a", "B", "C", "seq_idx")})
    return out


def _case(name):
    """(inputs, segments, dtype, chunk) of a named case."""
    if name in GENERAL:
        batch, T, H, P, N, seg, lengths, D, init, dtype, chunk = GENERAL[name]
    else:
        (batch, T, H, N, seg, lengths, D, init), P, dtype, chunk = CASES[name], 64, "bf16", 256
    assert sum(seg) == T
    d = make_custom(batch, T, H, P, N, 1, dtype, seed=4000 + len(name), has_D=D, has_init=init,
                    lengths=lengths)
    return d, seg, dtype, chunk


def _run_threads(d, seg, dtype="bf16", chunk=256):
    from mamba_ssd_layer_chunked_b200.sp import ssd_fwd_sp
    g = to_device(d, dtype)
    parts = _segments(g, seg)
    group = ThreadGroup(len(seg))
    out = [None] * len(seg)
    errors = []
    nseq = d["nseq"] if d["seq_idx"] is not None else None

    def rank_main(r):
        try:
            ag, ar = group.collectives(r)
            p = parts[r]
            out[r] = ssd_fwd_sp(p["X"], p["log_a"], p["B"], p["C"], chunk, rank=r, all_gather=ag, all_reduce_sum=ar,
                                D=g["D"], init_states=g["init_states"], seq_idx=p["seq_idx"], nseq=nseq)
        except BaseException as e:  # reported below
            errors.append(e)
            group.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(len(seg))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    if errors:
        raise errors[0]
    torch.cuda.synchronize()
    Y = torch.cat([o[0] for o in out], dim=1).float().cpu().numpy().astype(np.float64)
    finals = [o[1].cpu().numpy().astype(np.float64) for o in out]
    return Y, finals


@pytest.mark.parametrize("name", sorted(CASES) + sorted(GENERAL))
def test_sp_emulated_ranks_match_the_whole_sequence(name):
    d, seg, dtype, chunk = _case(name)
    Y, finals = _run_threads(d, seg, dtype, chunk)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU[dtype], "Y")
    for r, F in enumerate(finals):
        assert_close(F, Fr, TAU[dtype], f"final_states on rank {r}")
        assert np.array_equal(F, finals[0]), "ranks disagree on the final states"


def _last_piece_start(seq_row, a, b):
    if seq_row is None:
        return a
    last = seq_row[b - 1]
    return a + int(np.argmax(seq_row[a:b] == last))


@pytest.mark.parametrize("name", ["varlen_boundary_at_segment_edge", "three_ragged_segments", "skipped_ids",
                                  "f32_tiny_shape_reset", "bf16_N256_varlen", "bf16_P32_three_ranks"])
def test_sp_summary_is_the_state_after_the_last_piece(name):
    ssd = _ssd()
    d, seg, dtype, chunk = _case(name)
    g = to_device(d, dtype)
    parts = _segments(g, seg)
    bounds = np.cumsum([0] + list(seg))
    nseq = d["nseq"] if d["seq_idx"] is not None else 1
    batch, H = d["X"].shape[0], d["X"].shape[2]
    for r, p in enumerate(parts):
        loc, dec, ids = ssd.sp_summary(p["X"], p["log_a"], p["B"], seq_idx=p["seq_idx"], nseq=nseq, chunk=chunk)
        torch.cuda.synchronize()
        a, b = int(bounds[r]), int(bounds[r + 1])
        for bb in range(batch):
            row = None if d["seq_idx"] is None else d["seq_idx"][bb]
            st = _last_piece_start(row, a, b)
            sl = slice(bb, bb + 1), slice(st, b)
            _, Fr = oracle.ssd_reference(d["X"][sl], d["log_a"][sl], d["B"][sl], d["C"][sl])
            assert_close(loc[bb].cpu().numpy().astype(np.float64), Fr[0, 0], TAU[dtype], f"loc r={r} b={bb}")
            dref = np.exp(d["log_a"][bb, st:b].astype(np.float64).sum(axis=0))
            # an fp32 sum of the piece's log a: relative error ~1e-6 of |sum| in the exponent
            assert_close(dec[bb].cpu().numpy().astype(np.float64), dref, 1e-4, f"dec r={r} b={bb}", atol=1e-30)
            want = (0, 0) if row is None else (int(row[a]), int(row[b - 1]))
            assert tuple(ids[bb].tolist()) == want


def _draw_sp(i):
    """Random sequence-parallel problem i: (inputs, segments, dtype, chunk)."""
    rng = np.random.default_rng(5100 + i)
    dtype = "bf16" if rng.random() < 0.7 else "f32"
    b = int(rng.integers(1, 3))
    T = int(rng.integers(64, 1500))
    H = int(rng.choice([2, 4, 6]))
    P = int(rng.choice([32, 64, 64]))
    N = int(rng.choice([16, 64, 128, 128, 256]))
    Q = int(rng.choice([64, 128, 256]))
    R = int(rng.integers(2, 5))
    cuts = np.sort(rng.choice(np.arange(1, T), size=R - 1, replace=False))
    seg = np.diff(np.concatenate([[0], cuts, [T]])).astype(int).tolist()
    lengths = None
    if rng.random() < 0.6:
        nseq = int(rng.integers(1, 6))
        lengths = [np.diff(np.concatenate([[0], np.sort(rng.integers(0, T + 1, size=nseq - 1)), [T]])).astype(int).tolist()
                   for _ in range(b)]
    nseq = None if lengths is None else max(len(r) for r in lengths)
    d = make_custom(b, T, H, P, N, 1, dtype, seed=int(rng.integers(0, 10000)), has_D=str(rng.choice(["none", "normal"])),
                    has_init=bool(rng.random() < 0.5), lengths=lengths, nseq=nseq)
    return d, seg, dtype, Q


@pytest.mark.parametrize("i", range(12))
def test_sp_random_problem(i):
    d, seg, dtype, Q = _draw_sp(i)
    Y, finals = _run_threads(d, seg, dtype, Q)
    Yr, Fr = run_oracle(d)
    assert_close(Y, Yr, TAU[dtype], f"Y (segments {seg})")
    for r, F in enumerate(finals):
        assert_close(F, Fr, TAU[dtype], f"final_states on rank {r} (segments {seg})")
