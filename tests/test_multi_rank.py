"""Host logic of the multi-GPU bench on CPU: two gloo ranks.

The path shards by batch: each rank decodes its own batch, with no
collective on the data path, and the job's time is the slowest rank's
(weak scaling). These tests check the parts that do not need a GPU:
- the ranks draw distinct, reproducible batches;
- the max-over-ranks reduction gives every rank the same job time;
- the whole-job throughput counts every rank's bytes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = bench.rank_workload(rank)
        # a small batch of the rank's own workload (same seed recipe)
        small = bench.W.scaled(cfg, B=1, T_cap=64)
        inp = bench.W.make_inputs(small)
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slower one
        job_ms = bench.max_over_ranks(local_ms)
        value = bench.job_throughput(1_000_000, world, 4, job_ms)
        out[rank] = {"seed": cfg.seed, "k_sum": float(inp["k"].float().sum()), "job_ms": job_ms, "value": value}
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_batches_and_agree_on_time():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["k_sum"] != res[1]["k_sum"]                    # distinct batches
    assert res[0]["job_ms"] == res[1]["job_ms"] == 15.0          # slowest rank
    # 2 ranks x 4 steps x 1 MB over 15 ms
    assert res[0]["value"] == pytest.approx(2 * 4 * 1e6 / 15e-3 / 1e9)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(2e9, 1, 1, 1000.0) == pytest.approx(2.0)
    a, b = bench.rank_workload(0), bench.rank_workload(0)
    assert a.seed == b.seed                                       # reproducible
