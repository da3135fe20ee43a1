"""The multi-rank timing path of bench.py on CPU: two gloo ranks.

Replicas share no data-path collective; the only exchange is the max over ranks
of each device time, and the whole-job value is every rank's tokens over that
slowest time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    mine = [10.0 + 5.0 * rank, 3.0 - rank]            # ms: rank 1 is slower in the first value
    red = bench.reduce_over_ranks(torch, mine, "cpu")
    out[rank] = red + [bench.replica_value(32, world, red[0])]
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_sum_tokens():
    world = 2
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        for rank in range(world):
            assert out[rank][:2] == [15.0, 3.0]
            assert out[rank][2] == pytest.approx(32 * 2 / 0.015)


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(torch, [1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.overlap_efficiency(10.0, 8.0, 4.0) == 0.5
    assert bench.overlap_efficiency(8.0, 8.0, 4.0) == 1.0
    assert bench.overlap_efficiency(20.0, 8.0, 4.0) == 0.0
