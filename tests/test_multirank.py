"""The multi-replica path of bench.py on CPU: two gloo ranks with different step
times must both report the slowest rank's time and the whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = 100.0 + 10.0 * rank          # rank 1 is slower
    ms_e2e = 120.0 - 10.0 * rank      # rank 0 is slower end to end
    out = bench.aggregate_ranks(ms, ms_e2e, 1.0e14, world, dist)
    q.put((rank, out))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        ms, ms_e2e, value, value_e2e = res[rank]
        assert ms == 110.0 and ms_e2e == 120.0
        assert value == pytest.approx(2 * 1.0e14 / 0.110 / 1e12)
        assert value_e2e == pytest.approx(2 * 1.0e14 / 0.120 / 1e12)


def test_single_rank_needs_no_process_group():
    ms, ms_e2e, value, _ = bench.aggregate_ranks(50.0, 60.0, 1.0e14, 1)
    assert (ms, ms_e2e) == (50.0, 60.0) and value == pytest.approx(2000.0)
