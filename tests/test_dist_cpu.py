"""The multi-process plumbing of bench.py on CPU: two gloo ranks, the
max-over-ranks timing and the whole-job throughput (units of all ranks over
the slowest rank's time). No GPU and no data-path collective are involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        t = 0.5 + rank  # rank 1 is the slow one
        mx = bench.reduce_max(t)
        value, tmax = bench.aggregate(1000.0, t)
        out.put((rank, ws, r, local, mx, value, tmax))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_time_as_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, ws, r, local, mx, value, tmax in res:
        assert (ws, r, local) == (2, rank, rank)
        assert mx == 1.5 and tmax == 1.5          # max over ranks
        assert value == pytest.approx(2 * 1000.0 / 1.5)  # all ranks' units / slowest time


def test_single_process_helpers_are_identity():
    assert bench.reduce_max(3.0) == 3.0
    value, t = bench.aggregate(10.0, 2.0)
    assert (value, t) == (5.0, 2.0)
