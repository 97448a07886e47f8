"""The multi-rank path of bench.py on CPU with the gloo backend (world size 2):
the max-over-ranks timing reduction and the whole-job weak-scaling value.
(Ranks run independent replicas of the workload; the only collectives are
the barrier and this reduction.)"""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    per_rank_ms = [2.0, 3.5][rank]
    ms_max = bench.max_over_ranks(per_rank_ms, torch.device("cpu"))
    dist.barrier()
    value = bench.weak_scaling_value(1e12, world, ms_max)
    q.put((rank, ms_max, value))
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, value in res:
        assert ms_max == 3.5                      # the slowest rank's time, on every rank
        assert value == pytest.approx(2e12 / 3.5e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1.25, torch.device("cpu")) == 1.25
    assert bench.weak_scaling_value(10.0, 1, 1.0) == pytest.approx(1e4)
