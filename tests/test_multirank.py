"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

On N GPUs every rank runs its own batch of independent sequences (no
collective on the data path); the only cross-rank steps are the barriers
around the timed region and the maximum of the per-rank times.  These tests
exercise exactly those steps with two gloo ranks.
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    import hstu_inputs as hi
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        dist.barrier()
        # per-rank elapsed times: the reported time is the maximum over ranks
        t = bench.reduce_max(1.5 + rank, world, device="cpu")
        # every rank draws its own independent batch of the same workload shape
        spec = hi.workload("tiny")
        inp = hi.make_inputs(spec, seed=bench.rank_seed(0, rank))
        checksum = float(inp.q.double().sum())
        sums = [None] * world
        dist.all_gather_object(sums, checksum)
        out[rank] = (t, sums)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_batches():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 2.5          # max over ranks of 1.5 and 2.5
    sums = out[0][1]
    assert sums == out[1][1]
    assert sums[0] != sums[1]                      # ranks hold different batches


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.25, 1) == 3.25
    assert bench.rank_seed(7, 0) == 7 and bench.rank_seed(7, 3) != 7
