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


# ---- expert parallelism: partition and sum on gloo ranks ---------------------------

def _ep_rank_main(rank, world, port, out):
    """One rank of the expert-parallel layer, computed with the oracle's
    per-expert functions on the CPU: the slots whose expert this rank owns
    (the library's moe_ep_range), the shared expert on rank 0 only, then the
    sum over ranks by all-reduce."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np

    import oracle
    import routed_expert_ffn_05_b200 as M
    import synth
    cfg = synth.LayerConfig("ep", T=6, d=256, F=512, E=8, k=2, Fs=256)
    x, wr = synth.make_x(cfg), synth.make_router(cfg)
    q = {t: [oracle.mxfp4_quantize(synth.expert_weight_f32(cfg, 0, e, t)) for e in range(cfg.E)]
         for t in (synth.W1, synth.W3, synth.W2)}
    stack = lambda t, i: np.stack([q[t][e][i] for e in range(cfg.E)])
    ora = oracle.LayerWeights(cfg, stack(synth.W1, 0), stack(synth.W1, 1), stack(synth.W3, 0), stack(synth.W3, 1),
                              stack(synth.W2, 0), stack(synth.W2, 1), *synth.shared_weights_bf16(cfg), wr=wr)
    idx, w = oracle.topk_softmax(oracle.router_logits(x, wr), cfg.k)
    b, e = M.moe_ep_range(cfg.E, rank, world)
    y = np.zeros((cfg.T, cfg.d))
    for t in range(cfg.T):
        for j in range(cfg.k):
            if b <= idx[t, j] < e:
                y[t] += float(w[t, j]) * oracle.expert_ffn_token(ora, int(idx[t, j]), x[t])
        if rank == 0:
            y[t] += oracle.shared_ffn_token(ora, x[t])
    yt = torch.from_numpy(y)
    dist.all_reduce(yt, op=dist.ReduceOp.SUM)
    _, _, ref = oracle.layer_tokens(ora, x, np.arange(cfg.T, dtype=np.int32))
    out[rank] = (b, e, yt.numpy(), ref)
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_partition_and_sum(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_ep_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    import numpy as np
    ranges = [out[r][:2] for r in range(world)]
    owned = np.concatenate([np.arange(b, e) for b, e in ranges])
    np.testing.assert_array_equal(np.sort(owned), np.arange(8))        # every expert exactly once
    assert all(e - b in (8 // world, 8 // world + 1) for b, e in ranges)  # contiguous, balanced
    for r in range(world):
        np.testing.assert_array_equal(out[r][2], out[0][2])            # every rank holds the same sum
    ref = out[0][3]
    assert np.abs(out[0][2] - ref).max() <= 1e-5 * np.abs(ref).max()  # = the whole layer
