"""Benchmark of the quantized-KV decode path on B200.

One step = one pass of the whole path over one batch of the
Llama-3.1-8B-shaped workload (B16, 32 query / 8 KV heads, head_dim 128,
context 8192, group 64, K6V4, 1% heavy hitters):

  quantize   lkv_quantize_kv     bf16 K, V -> K6 / V4 codes + (scale, zero)
  decode     lkv_decode_attention  sparse-V skip at tau = 1e-4 (one launch)
  classify   lkv_tier_classify   Zipf(1.1) previous-step mass, tau_low 1e-4, tau_high 1e-2
  repack     lkv_tier_repack     kept tokens -> K6/V6 and K6/V4 segments
  tiered     lkv_tiered_attention  decode over the kept tokens (one launch)

value = algorithmic HBM bytes of the step / step time (GB/s), timed with CUDA
events on the launching stream with L2 flushed before every step; each
kernel is also timed on its own for the roofline.  Multi-GPU: one process per
GPU, every rank runs its own batch (weak scaling, no collective on the data
path), value = all ranks' bytes / max-over-ranks time.

--impl reference times the CPU oracle (the reference arm) on a bounded sample
of the same workload.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from quantized_kv_cache_lkv_b200 import workloads as W  # noqa: E402

CFG_ID = 2
KB, VB = 6, 4
TAU_LOW, TAU_HIGH = 1e-4, 1e-2       # tier thresholds of the tiered-cache workload
METRIC = "quantized-KV decode attention: HBM GB/s (% of peak), KV tokens/s"
L2_FLUSH_BYTES = 512 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def traffic_table():
    """ncu DRAM bytes per launch recorded in profiles/ncu_traffic.txt, keyed by
    kernel; an entry only counts while the kernel source still has the hash
    it was captured with."""
    out = {}
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return out
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        if len(parts) >= 4:
            out[parts[0]] = (parts[1], float(parts[2]), parts[3])
    return out


# Sources each timed kernel is compiled from (an ncu traffic figure only
# counts while these files are unchanged).
CSRC = "quantized_kv_cache_lkv_b200/csrc/"
KERNEL_SOURCES = {
    "quantize": [CSRC + "quantize.cu", CSRC + "lkv_device.cuh"],
    "repack": [CSRC + "quantize.cu", CSRC + "lkv_device.cuh"],
    "classify": [CSRC + "tier.cu"],
    "decode": [CSRC + "fused_impl.cuh", CSRC + "fused_k6.cu", CSRC + "lkv_device.cuh"],
    "tiered": [CSRC + "fused_impl.cuh", CSRC + "fused_k6.cu", CSRC + "lkv_device.cuh"],
}


def source_hash(name):
    h = hashlib.sha1()
    for rel in KERNEL_SOURCES[name]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 7:
                continue
            try:
                sm.append(float(p[0]))
                mx = float(p[1])
            except ValueError:
                continue
            for n, v in zip(names, p[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def path_bytes(cfg, seq_lens, counts, skipped_rows, skipped_rows_tiered):
    """Algorithmic HBM bytes of each kernel of one step.

    quantize  per valid row: bf16 K and V read, K6 + V4 codes and both
              (scale, zero) rows written;
    decode    every K row (codes + sz), the V rows some head keeps, q and out;
    classify  mass of valid tokens read, the tier byte of every slot written,
              4 bytes per kept position, the counts;
    repack    per kept token: bf16 K and V read, its position, codes + sz written;
    tiered    K rows of the kept tokens, their V rows unless every head
              skips them, q and out, the counts.
    """
    D, ng, Hkv = cfg.D, cfg.D // cfg.G, cfg.Hkv
    B, Hq, T_cap = cfg.B if seq_lens is None else len(seq_lens), cfg.Hq, cfg.T_cap
    rows = int(np.asarray(seq_lens, np.int64).sum()) * Hkv
    k_row, v_row, sz = D * KB // 8, D * VB // 8, 8 * ng
    r6, r4 = D * 6 // 8, D * 4 // 8
    qo = B * Hq * D * (2 + 4)
    n2, n1 = int(np.asarray(counts)[..., 0].sum()), int(np.asarray(counts)[..., 1].sum())
    kept = n2 + n1
    by = {
        "quantize": rows * (2 * D * 2 + k_row + v_row + 2 * sz),
        "decode": rows * (k_row + sz) + (rows - skipped_rows) * (v_row + sz) + qo,
        "classify": rows * 4 + B * Hkv * T_cap + kept * 4 + B * Hkv * 8,
        "repack": kept * (2 * D * 2 + 4 + r6 + sz) + n2 * (r6 + sz) + n1 * (r4 + sz),
    }
    v_kept = n2 * (r6 + sz) + n1 * (r4 + sz)
    keep_frac = 1.0 - skipped_rows_tiered / kept if kept else 0.0
    by["tiered"] = kept * (r6 + sz) + int(round(v_kept * keep_frac)) + qo + B * Hkv * 8
    return by


# ----------------------------------------------------------------- ranks

def rank_workload(rank):
    """The batch rank `rank` decodes: the bench workload with its own seed, so
    the ranks process distinct, independent batches (weak scaling)."""
    base = W.CONFIGS[CFG_ID]
    return W.scaled(base, seed=base.seed + 1000 * rank)


def max_over_ranks(x, device=None):
    """Maximum of a float over all ranks (the job's time is the slowest
    rank's); every rank takes part, with or without a process group."""
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step, world, steps, max_ms):
    """Whole-job GB/s: the bytes all ranks moved over the slowest rank's time."""
    return bytes_per_rank_step * world * steps / (max_ms * 1e-3) / 1e9


# ----------------------------------------------------------------- the step

class Step:
    """Device buffers and the launches of one step of the path."""

    def __init__(self, cfg, inp, device):
        from quantized_kv_cache_lkv_b200 import buffers, lkv
        self.lkv = lkv
        self.cfg = cfg
        B, Hq, Hkv, D, T, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.G
        self.shape = (B, Hq, Hkv, D, T, G)
        d = {k: v.to(device) for k, v in inp.items()}
        self.d = d
        self.cache = buffers.alloc_cache(KB, VB, G, B, Hkv, T, D, device, zero=True)
        self.out = torch.empty(B, Hq, D, device=device)
        self.out2 = torch.empty(B, Hq, D, device=device)
        self.cnt = torch.zeros(2, dtype=torch.int64, device=device)
        self.cnt2 = torch.zeros(2, dtype=torch.int64, device=device)
        self.ws = buffers.alloc_workspace(lkv.lkv_decode_workspace_bytes((KB, VB, G), B, Hq, Hkv, T, D), device)
        self.ws2 = buffers.alloc_workspace(lkv.lkv_tiered_workspace_bytes(B, Hq, Hkv, T, D, G), device)
        self.tiers = buffers.alloc_tiers(B, Hkv, T, device, zero=True)
        self.A, self.Bs = buffers.alloc_segments(G, B, Hkv, T, D, device, zero=True)
        self.names = ["quantize", "decode", "classify", "repack", "tiered"]

    def launches(self, stream, events=None):
        L, c, d = self.lkv, self.cfg, self.d
        B, Hq, Hkv, D, T, G = self.shape
        s = stream.cuda_stream

        def mark(i):
            if events is not None:
                events[i].record(stream)
        mark(0)
        L.lkv_quantize_kv((KB, VB, G), B, Hkv, T, D, d["seq_lens"], d["k"], d["v"], self.cache["k_codes"],
                          self.cache["k_sz"], self.cache["v_codes"], self.cache["v_sz"], s)
        mark(1)
        L.lkv_decode_attention((KB, VB, G), B, Hq, Hkv, T, D, d["seq_lens"], d["q"], self.cache["k_codes"],
                               self.cache["k_sz"], self.cache["v_codes"], self.cache["v_sz"],
                               c.softmax_scale, c.tau, self.out, None, self.cnt, self.ws, self.ws.numel(), s)
        mark(2)
        t = self.tiers
        L.lkv_tier_classify(B, Hkv, T, d["seq_lens"], d["mass"], TAU_LOW, TAU_HIGH, t["tier"], t["counts"],
                            t["pos_a"], t["pos_b"], s)
        mark(3)
        L.lkv_tier_repack(B, Hkv, T, D, G, d["k"], d["v"], t["counts"], t["pos_a"], t["pos_b"], self.A,
                          self.Bs, s)
        mark(4)
        L.lkv_tiered_attention(B, Hq, Hkv, T, D, G, t["counts"], d["q"], self.A, self.Bs, c.softmax_scale,
                               0.0, self.out2, self.cnt2, self.ws2, self.ws2.numel(), s)
        mark(5)

    LAUNCHES_PER_STEP = 5    # quantize, decode, classify, repack, tiered: one kernel each

    def algorithmic_bytes(self):
        """Bytes each kernel must move, from the step's device results."""
        B, Hq, Hkv, D, T, G = self.shape
        sl = self.d["seq_lens"].cpu().numpy()
        counts = self.tiers["counts"].cpu().numpy()
        self.skipped_rows = int(self.cnt[1].item())
        by = path_bytes(self.cfg, sl, counts, self.skipped_rows, int(self.cnt2[1].item()))
        self.kept = (int(counts[..., 0].sum()), int(counts[..., 1].sum()), int(sl.astype(np.int64).sum()) * Hkv)
        return by

    def dense_decode_bytes(self):
        B, Hq, Hkv, D, T, G = self.shape
        rows = int(self.d["seq_lens"].sum().item()) * Hkv
        return rows * (D * (KB + VB) // 8 + 16 * (D // G)) + B * Hq * D * 6


def run_lkv(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    if dist:
        import datetime
        import torch.distributed as tdist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    from __graft_entry__ import build
    build()

    cfg = rank_workload(rank)
    inp = W.make_inputs(cfg, with_mass=True)
    step = Step(cfg, inp, device)
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def barrier():
        if dist:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        flush.zero_()
        step.launches(stream)
    barrier()
    n = len(step.names)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier()
        for i in range(args.steps):
            flush.zero_()                      # L2 flush, outside the timed region
            step.launches(stream, ev[i])
        barrier()
    per_kernel = {name: [] for name in step.names}
    step_ms = []
    for i in range(args.steps):
        for j, name in enumerate(step.names):
            per_kernel[name].append(ev[i][j].elapsed_time(ev[i][j + 1]))
        step_ms.append(ev[i][0].elapsed_time(ev[i][n]))
    total_ms = max_over_ranks(sum(step_ms), device)
    by = step.algorithmic_bytes()
    step_bytes = sum(by.values())
    value = job_throughput(step_bytes, world, args.steps, total_ms)
    kv_tokens = int(inp["seq_lens"].sum()) * world
    peak, peak_kind = peaks()

    # per-kernel roofline (algorithmic bytes / mean launch time)
    kern = {}
    for name in step.names:
        ms = statistics.mean(per_kernel[name])
        gbs = by[name] / (ms * 1e-3) / 1e9
        kern[name] = {"us": round(ms * 1e3, 2), "bytes": by[name], "gbs": round(gbs, 1),
                      "frac": round(gbs / peak, 4), "share": round(ms / statistics.mean(step_ms), 4)}
    dominant = max(step.names, key=lambda k: kern[k]["us"])
    traffic = traffic_table()

    def roofline(name):
        tr = traffic.get(name)
        t_bytes = None
        if tr and tr[0] == source_hash(name):
            t_bytes = tr[1]
        return {"bound": "hbm", "achieved": kern[name]["gbs"], "peak": peak, "unit": "GB/s",
                "frac": kern[name]["frac"], "traffic": t_bytes, "kernel": name,
                "peak_source": f"{peak_kind} hbm_gbs"}

    e2e = None
    if not args.no_e2e:   # every rank runs it; the job's time is the slowest rank's
        e2e = run_e2e(step, inp, device, stream, args)
        sec = max_over_ranks(e2e["seconds"], device)
        e2e["value"] = round(job_throughput(e2e["bytes"], world, e2e["steps"], sec * 1e3), 2)
    cpu = cpu_baseline(cfg, inp, args) if rank == 0 and world == 1 and not args.no_cpu else None

    if rank == 0:
        clk = clocks.summary()
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "head_dim": cfg.D,
                       "context": cfg.T_cap, "group": cfg.G, "k_bits": KB, "v_bits": VB, "tau": cfg.tau,
                       "heavy_hitters": cfg.hh_frac, "tier_tau_low": TAU_LOW, "tier_tau_high": TAU_HIGH,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": "flushed before every step (512 MiB write)",
                       "step": "quantize + decode + tier classify + repack + tiered decode"},
            "kv_tokens_per_s": round(kv_tokens * args.steps / (total_ms * 1e-3), 1),
            "roofline": roofline(dominant),
            "roofline_decode": roofline("decode"),
            "kernels": kern,
            "decode_skip": {"v_rows_skipped": step.skipped_rows, "rows": step.kept[2],
                            "frac": round(step.skipped_rows / max(step.kept[2], 1), 4),
                            "dense_bytes": step.dense_decode_bytes()},
            "tiers": {"v6": step.kept[0], "v4": step.kept[1], "rows": step.kept[2]},
            "gpu_launches": Step.LAUNCHES_PER_STEP * args.steps,
            "clocks": {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "e2e": {k: e2e[k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step")}
            if e2e else None,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_e2e(step, inp, device, stream, args):
    """The same step through the public API from pinned host memory: every
    step copies its inputs host->device and reads both outputs back."""
    host = {k: v.pin_memory() for k, v in inp.items()}
    h_out = torch.empty(step.out.shape, dtype=torch.float32).pin_memory()
    h_out2 = torch.empty(step.out2.shape, dtype=torch.float32).pin_memory()
    n = max(1, min(args.e2e_steps, args.steps))
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = 2 * h_out.numel() * 4
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(n + 1):
        if i == 1:
            torch.cuda.synchronize(device)
            start.record(stream)
        for k in host:
            step.d[k].copy_(host[k], non_blocking=True)
        step.launches(stream)
        h_out.copy_(step.out, non_blocking=True)
        h_out2.copy_(step.out2, non_blocking=True)
    end.record(stream)
    torch.cuda.synchronize(device)
    sec = start.elapsed_time(end) * 1e-3
    by = sum(step.algorithmic_bytes().values())
    return {"value": round(by * n / sec / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "seconds": sec, "bytes": by, "steps": n}


# ----------------------------------------------------------------- CPU oracle

def oracle_step(orc, cfg, sub):
    """One pass of the oracle over a sample: quantize, decode, tiers, repack,
    tiered attention.  Returns the algorithmic bytes of the sample."""
    k, v, q = W.bf16_bits(sub["k"]), W.bf16_bits(sub["v"]), W.bf16_bits(sub["q"])
    sl, mass = sub["seq_lens"].numpy(), sub["mass"].numpy()
    cache = orc.quantize_kv(KB, VB, cfg.G, k, v, sl)
    _, _, cnt = orc.decode_attention(KB, VB, cfg.G, sl, q, cache, cfg.softmax_scale, cfg.tau, want_mask=False)
    tier, counts, p2, p1 = orc.tier_classify(sl, mass, TAU_LOW, TAU_HIGH)
    A, Bs = orc.tier_repack(cfg.G, k, v, counts, p2, p1)
    _, cnt2 = orc.tiered_attention(cfg.G, counts, q, A, Bs, cfg.softmax_scale, 0.0)
    return sum(path_bytes(cfg, sl, counts, int(cnt[1]), int(cnt2[1])).values())


def oracle_sample(cfg, inp, n_seq):
    return {k: inp[k][:n_seq].contiguous() for k in ("q", "k", "v", "seq_lens", "mass")}


def cpu_baseline(cfg, inp, args):
    import oracle
    oracle.lib()
    target = args.cpu_seconds
    n_seq = 1
    t0 = time.perf_counter()
    by = oracle_step(oracle, cfg, oracle_sample(cfg, inp, n_seq))
    dt = time.perf_counter() - t0
    if dt < target / 2 and n_seq < cfg.B:
        n_seq = int(min(cfg.B, max(1, math.floor(target / max(dt, 1e-3)))))
        t0 = time.perf_counter()
        by = oracle_step(oracle, cfg, oracle_sample(cfg, inp, n_seq))
        dt = time.perf_counter() - t0
    # the whole batch may still be quick on a large host: repeat the pass
    sample = oracle_sample(cfg, inp, n_seq)
    passes, total_by, total_dt = 1, by, dt
    while total_dt < target:
        t0 = time.perf_counter()
        total_by += oracle_step(oracle, cfg, sample)
        total_dt += time.perf_counter() - t0
        passes += 1
    return {"value": round(total_by / total_dt / 1e9, 4), "unit": "GB/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"first {n_seq} of {cfg.B} sequences of {cfg.name}, {passes} oracle pass(es) "
                      f"(quantize + decode + tiers + repack + tiered), {total_dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.lib()
    cfg = W.CONFIGS[CFG_ID]
    inp = W.make_inputs(cfg, with_mass=True)
    # bounded sample per step so the whole run stays within a few minutes
    n_seq = 1
    sub = oracle_sample(cfg, inp, n_seq)
    for _ in range(args.warmup):
        oracle_step(oracle, cfg, sub)
    times, by = [], 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        by = oracle_step(oracle, cfg, sub)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = by * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "head_dim": cfg.D,
                   "context": cfg.T_cap, "group": cfg.G, "k_bits": KB, "v_bits": VB, "tau": cfg.tau,
                   "parallelism": "single", "sample_sequences": n_seq},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"first {n_seq} of {cfg.B} sequences per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lkv", "reference"], default="lkv")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_lkv(args)


if __name__ == "__main__":
    main()
