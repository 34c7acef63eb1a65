"""The N > 1 host path of bench.py on CPU: two gloo ranks reduce their step
times by max over ranks, the way the GPU run does over NCCL."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    dist = bench.dist_init(world, backend="gloo")
    r, w, _ = bench.dist_env()
    # each rank reports its own summed step time; the job's time is the slowest rank's
    mine = 10.0 + 5.0 * r
    got = bench.max_over_ranks(mine, w)
    bench.barrier(w)
    out[r] = got
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_useful_flop_count():
    import bench

    # the 4096^2 five-step call: 1.3746e12 triangle-counted FLOPs
    assert bench.useful_flops(4096, 4096, 5) == 5 * (4096 * 4096 * 4097 * 2 + 2 * 4096 ** 3)
    assert abs(bench.useful_flops(4096, 4096, 5) - 1.3746e12) / 1.3746e12 < 1e-4
