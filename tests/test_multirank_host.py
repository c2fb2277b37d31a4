"""The multi-rank host logic of bench.py on CPU: two gloo ranks, each with a
different measured time, must agree on the slowest one, and the whole-job
throughput counts every rank's bytes over that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    t = bench.max_over_ranks(1.0 + rank)        # rank 0: 1 s, rank 1: 2 s
    out[rank] = t
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert dict(out) == {0: 2.0, 1: 2.0}


def test_single_process_and_aggregate():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    # 2 ranks x 10 steps x 1e9 bytes in 2 s -> 10 GB/s
    assert bench.aggregate_gbs(10**9, 10, 2, 2.0) == pytest.approx(10.0)
