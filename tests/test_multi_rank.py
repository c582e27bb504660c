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
        value = bench.job_throughput(1_000_000, world, job_ms * 1e-3)
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
    # 2 ranks x 1 MB over the slowest rank's 15 ms
    assert res[0]["value"] == pytest.approx(2 * 1e6 / 15e-3 / 1e9)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(2e9, 1, 1.0) == pytest.approx(2.0)
    a, b = bench.rank_workload(0), bench.rank_workload(0)
    assert a.seed == b.seed                                       # reproducible


def test_decode_bytes_per_row():
    """Algorithmic bytes of the decode metric: for the Llama-3.1-8B-shaped
    K6V4 rows (D 128, group 64) a K row is 96 code bytes + 16 bytes of
    (scale, zero), a kept V row 64 + 16, and q (bf16) + out (f32) 6 bytes
    per (b, h, d)."""
    assert bench.decode_bytes(10, 4, 2, 32, 128, 64, 6, 4) == 10 * 112 + 4 * 80 + 2 * 32 * 128 * 6
    assert bench.quantize_bytes(3, 128, 64, 6, 4) == 3 * (512 + 96 + 64 + 32)


def test_reference_arm_prints_one_json_line():
    """The reference arm (the CPU oracle) runs without a GPU and prints the
    contract's line: impl, metric, value, unit, config of the GPU arm, a
    cpu_baseline describing the run and an e2e block with no host copies."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=root)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.W.CONFIGS[bench.CFG_MAIN].name
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
