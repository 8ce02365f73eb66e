"""The N > 1 replica path of bench.py on CPU: two gloo ranks.

bench.py --gpus N runs one independent replica per GPU (the layer partitions
by token batch, so no data-path collective exists): each rank times its own
batches, the job value is every rank's tokens over the slowest rank's time,
and the barrier / max-over-ranks plumbing is the only communication. This
test runs that plumbing with the gloo backend on two CPU processes.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # each rank "measures" a different time; everyone must agree on the slowest
    my_seconds = 1.0 + rank * 0.5
    bench.barrier(torch, world)
    slowest = bench.max_over_ranks(torch, world, my_seconds)
    value = bench.job_value(world, 8, 10, slowest)
    seeds = [bench.batch_index(rank, b) for b in range(bench.NBATCH)]
    out[rank] = (slowest, value, seeds)
    dist.destroy_process_group()


def test_two_rank_replicas_agree_on_slowest_rank():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    slowest = {r: out[r][0] for r in range(world)}
    assert slowest == {0: 1.5, 1: 1.5}                 # max over ranks, on every rank
    assert out[0][1] == out[1][1] == world * 8 * 10 / 1.5  # whole-job tokens over the slowest time
    s0, s1 = set(out[0][2]), set(out[1][2])
    assert len(s0) == len(s1) == 8 and not (s0 & s1)   # replicas never share a batch


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(torch, 1, 3.0) == 3.0
    assert bench.job_value(1, 8, 10, 2.0) == 40.0
