"""The multi-rank path of bench.py on CPU: two gloo ranks on 127.0.0.1 check that device times
are reduced to their maximum over ranks and that throughput counts every rank's work (the
replicas share no data, so these reductions are the only collectives of a run)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (r + 1) ms for the step and 10 - r ms for the stage
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], torch.device("cpu"))
        rate = bench.job_rate(world, 32, got[0])
        dist.barrier()
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_reduce_to_the_slowest_and_count_all_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=90) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, got, rate in res:
        assert got == [2.0, 10.0]                    # max over ranks of each value
        assert rate == pytest.approx(2 * 32 / 2e-3)  # both ranks' queries over the slowest time


def test_single_process_reduction_is_the_identity():
    assert bench.max_over_ranks([3.5, 1.0], torch.device("cpu")) == [3.5, 1.0]
    assert bench.job_rate(1, 32, 0.1) == pytest.approx(320000.0)
