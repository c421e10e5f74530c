"""Host side of the multi-GPU bench path on CPU: two gloo ranks (no GPU).

With N GPUs the bench runs N independent replicas of the layer; the only
cross-rank steps are a barrier and a MAX reduction of the timed region, and
the job throughput is all ranks' tokens over the slowest rank's time.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(100.0 + 50.0 * rank, world)   # rank 1 is slower
        v = bench.job_throughput(8192, 10, t, world)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_job_throughput(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t, v in res:
        assert t == 150.0                                   # every rank sees the slowest
        assert v == pytest.approx(world * 8192 * 10 / 0.150)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(100, 2, 1000.0, 1) == 200.0
