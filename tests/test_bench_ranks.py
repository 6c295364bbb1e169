"""Multi-rank host logic of bench.py on CPU: two gloo ranks, weak-scaling shards.

Each rank times its own batch; the job time is the max over ranks and the
throughput counts every rank's crops. Shards of a workload share shapes and
draw different data.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from prompt_conditioned_keypoint_b200 import synthetic as S


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own = [0.25, 0.75][rank]                      # rank 1 is the slow one
        m = bench.max_over_ranks(own, dist, "cpu")
        results[rank] = (m, bench.job_throughput(world, 64, 10, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    world, port = 2, _free_port()
    results = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, results), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        m, value = results[r]
        assert m == 0.75                              # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 64 * 10 / 0.75)


def test_single_rank_needs_no_group():
    assert bench.max_over_ranks(1.5) == 1.5
    assert bench.job_throughput(1, 64, 100, 2.0) == 3200.0


@pytest.mark.parametrize("cfg", [2, 4])
def test_shards_share_shape_and_differ_in_data(cfg):
    a, b = S.make_config(cfg, crops=[0, 1], shard=0), S.make_config(cfg, crops=[0, 1], shard=1)
    assert a.feat.shape == b.feat.shape and a.mask.shape == b.mask.shape
    assert not np.array_equal(a.feat, b.feat)
    again = S.make_config(cfg, crops=[0, 1], shard=1)
    assert np.array_equal(again.feat, b.feat) and np.array_equal(again.mask, b.mask)
