"""Host-side logic of the N > 1 bench path, run as two gloo ranks on the CPU:
the max-over-ranks timing reduction and the whole-job throughput."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms, world)
    value = bench.job_throughput(1000.0, world, ms_max)
    bench.barrier(world)
    out[rank] = (ms_max, value)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    ms_max, value = out[0]
    assert ms_max == 15.0
    assert value == pytest.approx(1000.0 * 2 / 0.015)
