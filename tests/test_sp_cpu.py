"""The sequence-parallel driver over two gloo ranks on CPU.

The driver (mamba_ssd_layer_chunked_b200.sp.ssd_fwd_sp) is run as it runs
over NCCL, with torch.distributed collectives, but with its four compute steps
given by the fp64 oracle instead of the library's kernels (there is no GPU
here): the summary is the oracle's state after the segment's last sequence
piece, the combine and the ownership of final states restate the rules that
the kernels implement, and the forward pass is the oracle's recurrence. Each
rank's Y and the assembled final states must equal the oracle on the whole
sequence (fp64 throughout, so to ~1e-12).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from workloads import make_custom

CASES = {
    "one_sequence": (2, 300, 3, 16, 16, None, True),
    "boundary_at_the_cut": (2, 300, 3, 16, 16, [[100, 50, 150], [300]], True),
    "skipped_ids": (1, 300, 2, 16, 16, [[0, 90, 0, 210, 0]], True),
}
CUT = 150  # rank 0: tokens [0, 150), rank 1: [150, 300)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(name):
    batch, T, H, P, N, lengths, init = CASES[name]
    return make_custom(batch, T, H, P, N, 1, "f32", seed=77, has_D="normal", has_init=init, lengths=lengths)


class OracleOps:
    """The driver's compute steps from the oracle (fp64, torch CPU tensors)."""

    @staticmethod
    def summary(X, log_a, B, seq_idx, nseq, chunk):
        Xn, la, Bn = X.numpy(), log_a.numpy(), B.numpy()
        batch, T, H, P = Xn.shape
        N = Bn.shape[3]
        loc = np.zeros((batch, H, N, P))
        dec = np.zeros((batch, H))
        ids = np.zeros((batch, 2), dtype=np.int32)
        for b in range(batch):
            row = None if seq_idx is None else seq_idx[b].numpy()
            st = 0 if row is None else int(np.argmax(row == row[-1]))
            _, F = oracle.ssd_reference(Xn[b:b + 1, st:], la[b:b + 1, st:], Bn[b:b + 1, st:], Bn[b:b + 1, st:])
            loc[b] = F[0, 0]
            dec[b] = np.exp(la[b, st:].astype(np.float64).sum(axis=0))
            ids[b] = (0, 0) if row is None else (row[0], row[-1])
        return torch.from_numpy(loc), torch.from_numpy(dec), torch.from_numpy(ids)

    @staticmethod
    def combine(X, B, g_loc, g_dec, g_ids, rank, init_states, nseq, chunk):
        batch, _, H, P = X.shape
        N = B.shape[3]
        init = (torch.zeros((batch, nseq, H, N, P), dtype=torch.float64) if init_states is None
                else init_states.clone())
        out = init.clone()
        for b in range(batch):
            first = int(g_ids[rank, b, 0])
            if rank == 0 or int(g_ids[rank - 1, b, 1]) != first:
                continue
            E = torch.zeros((H, N, P), dtype=torch.float64)
            for j in range(rank):
                fj, lj = int(g_ids[j, b, 0]), int(g_ids[j, b, 1])
                carried = j > 0 and fj == lj and int(g_ids[j - 1, b, 1]) == fj
                start = E if carried else init[b, lj]
                E = g_dec[j, b][:, None, None] * start + g_loc[j, b]
            out[b, first] = E
        return out

    @staticmethod
    def forward(X, log_a, B, C, chunk, D, init_local, seq_idx, nseq, return_final_states):
        Y, F = oracle.ssd_reference(X.numpy(), log_a.numpy(), B.numpy(), C.numpy(),
                                    None if D is None else D.numpy(), init_local.numpy(),
                                    None if seq_idx is None else seq_idx.numpy(), nseq=nseq)
        return torch.from_numpy(Y), torch.from_numpy(F)

    @staticmethod
    def own_finals(X, B, final, g_ids, rank, nseq, chunk):
        R = g_ids.shape[0]
        for b in range(final.shape[0]):
            for s in range(nseq):
                owner = 0
                for j in range(R):
                    if int(g_ids[j, b, 0]) <= s:
                        owner = j
                if owner != rank:
                    final[b, s] = 0
        return final


def _rank_main(rank, world, port, name, out):
    import torch.distributed as dist
    from mamba_ssd_layer_chunked_b200.sp import ssd_fwd_sp, torch_collectives
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = _inputs(name)
        sl = slice(0, CUT) if rank == 0 else slice(CUT, None)
        t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a[:, sl]))
        init = None if d["init_states"] is None else torch.from_numpy(d["init_states"].astype(np.float64))
        D = torch.from_numpy(d["D"].astype(np.float64))
        ag, ar = torch_collectives()
        Y, F = ssd_fwd_sp(t(d["X"]), t(d["log_a"]), t(d["B"]), t(d["C"]), 64, rank=rank, all_gather=ag,
                          all_reduce_sum=ar, D=D, init_states=init, seq_idx=t(d["seq_idx"]),
                          nseq=d["nseq"] if d["seq_idx"] is not None else None, ops=OracleOps)
        out.put((rank, Y.numpy(), F.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("name", sorted(CASES))
def test_two_gloo_ranks_give_the_whole_sequence(name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, name, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (Y, F)) for r, Y, F in (q.get(timeout=150) for _ in procs))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    d = _inputs(name)
    Yr, Fr = oracle.ssd_reference(d["X"], d["log_a"], d["B"], d["C"], d["D"], d["init_states"], d["seq_idx"],
                                  nseq=d["nseq"])
    Y = np.concatenate([res[0][0], res[1][0]], axis=1)
    np.testing.assert_allclose(Y, Yr, rtol=0, atol=1e-10 * np.abs(Yr).max())
    for r in (0, 1):
        np.testing.assert_allclose(res[r][1], Fr, rtol=0, atol=1e-10 * np.abs(Fr).max())
