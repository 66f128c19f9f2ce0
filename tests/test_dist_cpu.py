"""The N>1 path of bench.py on CPU: two gloo ranks (weak scaling over sequences).

Every rank holds its own sequences (no collective on the data path); the only
collectives are the barrier and the max-over-ranks reduction of the step time,
which these tests run on the host.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # per-rank step times; every rank must see the maximum
        ms = 1.0 + 0.5 * rank
        ms_max = bench.max_over_ranks(ms, dist)
        bench.barrier(dist)
        # this rank's sequences: its own draws of the workload recipe
        w = synth.scaled(bench.rank_workload("csa_flash_128k", rank), B=2, L=4 * 300, top_k=16)
        inp = synth.decode_layer_inputs(w, 0)
        sh = list(bench.shard(rank, world, w.B))
        out[rank] = dict(ms_max=ms_max, shard=sh, q_sum=float(np.abs(inp["Q"]).sum()),
                         seed=w.seed, value=bench.job_value(ms_max, w.B, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    # max over ranks reaches every rank
    assert res[0]["ms_max"] == res[1]["ms_max"] == pytest.approx(1.5)
    # disjoint shards covering 0 .. world*B-1
    assert res[0]["shard"] == [0, 1] and res[1]["shard"] == [2, 3]
    # different sequences per rank, rank 0 = the one-GPU draws
    assert res[0]["seed"] == synth.WORKLOADS["csa_flash_128k"].seed
    assert res[0]["seed"] != res[1]["seed"] and res[0]["q_sum"] != res[1]["q_sum"]
    # whole-job throughput: both ranks' sequences in the slowest rank's time
    assert res[0]["value"] == pytest.approx(2 * 2 / 1.5e-3)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.0, None) == 3.0
    assert list(bench.shard(0, 1, 4)) == [0, 1, 2, 3]
    assert bench.job_value(2.0, 4, 1) == pytest.approx(2000.0)
    assert bench.rank_workload("pro_pair_1m", 0) is synth.WORKLOADS["pro_pair_1m"]
