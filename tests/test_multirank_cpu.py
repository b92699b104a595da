"""The benchmark's multi-rank host logic on CPU with two gloo ranks: every rank runs its own
batch (weak scaling), the job time is the slowest rank's, and the only collective is the
scalar max over ranks.  No GPU is touched."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [10.0, 25.0][rank]            # rank 1 is the slow one
        rate, ms = bench.whole_job_rate(16384, 20, local_ms, world, device="cpu")
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, rate, ms))
        if rank == 0:
            out.put(gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_the_slowest_and_count_every_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, rate, ms in res:
        assert ms == 25.0                                    # the max over ranks, on every rank
        assert rate == pytest.approx(2 * 16384 * 20 / 0.025)  # both ranks' tokens / slowest time


def test_single_rank_needs_no_collective():
    import bench
    rate, ms = bench.whole_job_rate(100, 4, 8.0, 1, device="cpu")
    assert ms == 8.0 and rate == pytest.approx(100 * 4 / 0.008)
