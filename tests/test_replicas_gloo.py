"""Host logic of the multi-GPU bench path (replicas, max-over-ranks timing)
on CPU with gloo, world size 2."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 10.0 + 5.0 * rank        # rank 1 is the slow one
    got = bench.max_over_ranks(ms, world, torch.device("cpu"))
    val = bench.job_value(1000, world, got)
    q.put((rank, got, val))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, val in res:
        assert got == 15.0
        assert val == pytest.approx(1000 * 2 / 15e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.job_value(10, 1, 1.0) == pytest.approx(1e4)
