"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU.

With N GPUs each rank runs its own batch of the workload (the query heads are
independent, so nothing is exchanged on the data path); the ranks only agree on
a barrier and on the slowest rank's time, which sets the reported throughput.
"""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = bench.init_dist(world, "gloo")
    dev = torch.device("cpu")
    bench.barrier(d, dev)
    local_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    slowest = bench.max_over_ranks(local_ms, d, dev)
    seeds = bench.rank_seed(1002, rank)
    out[rank] = (slowest, seeds)
    bench.barrier(d, dev)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_slowest_time_and_draw_distinct_batches():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:   # no fork of a multi-threaded process
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1]


def test_single_rank_needs_no_process_group():
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_whole_job_value_counts_every_rank():
    from attn_inputs import get_workload
    w = get_workload("cfg2")
    # value = world * flops * steps / slowest time: two ranks at the same speed double it
    one = 1 * w.flops * 10 / 1.0
    two = 2 * w.flops * 10 / 1.0
    assert two == pytest.approx(2 * one)
