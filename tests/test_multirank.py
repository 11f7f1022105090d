"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
the step time is the maximum over ranks and the job value counts every
rank's work (weak scaling, one replica per rank)."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms_local = [2.0, 3.5][rank]
        value, ms = bench.job_throughput(1000.0, ms_local, world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, value, ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms in results:
        assert ms == pytest.approx(3.5)
        assert value == pytest.approx(1000.0 * 2 / 3.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    value, ms = bench.job_throughput(500.0, 4.0, 1, torch.device("cpu"))
    assert ms == 4.0 and value == pytest.approx(500.0 / 4e-3)
