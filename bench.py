"""Benchmark of the quantized-KV decode path on B200.

Headline (`value`): the decode call, lkv_decode_attention, on the
Llama-3.1-8B-shaped workload (B16, 32 query / 8 KV heads, head_dim 128,
context 8192, group 64, K6V4, 1% heavy hitters, sparse-V skip at tau 1e-4):
its algorithmic HBM bytes (every K row and (scale, zero) row, the V rows some
head keeps, q and out) over the median of its device times, in GB/s.

Each timed step runs the whole path once on that workload, with L2 flushed
(a 512 MiB write) before every kernel, outside the kernel's event pair:

  quantize   lkv_quantize_kv       bf16 K, V -> K6 / V4 codes + (scale, zero)
  decode     lkv_decode_attention  one launch, sparse-V skip at tau = 1e-4
  classify   lkv_tier_classify     Zipf(1.1) previous-step mass, tau_low 1e-4, tau_high 1e-2
  repack     lkv_tier_repack       kept tokens -> K6/V6 and K6/V4 segments
  tiered     lkv_tiered_attention  decode over the kept tokens (one launch)

and the step's figures sit under "step".  At one GPU the other workloads
follow under their own keys, each timed the same way (median over the timed
steps, L2 flushed before every launch):

  long_context  B1, context 131072, tau 1e-5, 0.1% heavy hitters: decode, and
                quantize of the full 131072-token bf16 K/V;
  bit_sweep     B64, ragged context uniform in [512, 4096], group 32: decode
                per (k_bits, v_bits) in K8V8, K6V4, K4V4, K4V2, with the
                measured compression ratio against the bit-count formula and
                the rel-L2 error against fp64 attention over the unquantized
                bf16 cache (computed with torch in float64 on the device);
  tiered        B32, context log-uniform in [1024, 32768], Zipf(1.1) mass:
                classify, repack and tiered decode, with the tiered cache's
                compression ratio.

stream: the same decode call back to back, rotating over four copies of the
quantized cache (inputs larger than L2 instead of a flush between calls);
events around each block of calls, per-call time = block time / calls, median
over the blocks.  It is the call's throughput in a decode loop, where the
launch latency overlaps the previous call and the code stays resident; the
headline keeps the isolated, flushed figure.

--call NAME times only one call of the step (after one untimed pass of the
whole step), the way the ncu commands under profiles/ capture it.

e2e is a decode loop through the public API with host buffers: every step
copies q and the new token's K/V (plus positions and lengths) host->device in
one copy from a pinned staging buffer, appends the token (lkv_append_kv),
decodes, and reads out and the skip counts back device->host in one copy;
value = the decode + append algorithmic bytes over the loop's device time.

Multi-GPU: one process per GPU, every rank decodes its own batch (weak
scaling, no collective on the data path), value = all ranks' decode bytes /
the max-over-ranks median time.

--impl reference times the CPU oracle (the reference arm) on the same
workload and metric.
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

CFG_MAIN, CFG_LONG, CFG_SWEEP, CFG_TIER = 2, 3, 4, 5
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
FUSED = [CSRC + "fused_impl.cuh", CSRC + "mma_k.cuh", CSRC + "fused_k6.cu", CSRC + "lkv_device.cuh"]
KERNEL_SOURCES = {
    "quantize": [CSRC + "quantize.cu", CSRC + "lkv_device.cuh"],
    "repack": [CSRC + "quantize.cu", CSRC + "lkv_device.cuh"],
    "classify": [CSRC + "tier.cu"],
    "decode": FUSED,
    "tiered": FUSED,
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


# ----------------------------------------------------------------- algorithmic bytes

def sz_bytes(D, G):
    return 8 * (D // G)


def quantize_bytes(rows, D, G, kb, vb):
    """bf16 K and V read, K and V codes and both (scale, zero) rows written."""
    return rows * (2 * D * 2 + D * kb // 8 + D * vb // 8 + 2 * sz_bytes(D, G))


def decode_bytes(rows, v_rows_kept, B, Hq, D, G, kb, vb):
    """Every K row and its (scale, zero), the V rows some head keeps, q and out."""
    return rows * (D * kb // 8 + sz_bytes(D, G)) + v_rows_kept * (D * vb // 8 + sz_bytes(D, G)) + B * Hq * D * 6


def classify_bytes(rows, B, Hkv, T_cap, kept):
    """Mass of valid tokens read, the tier byte of every slot, 4 bytes per kept position, the counts."""
    return rows * 4 + B * Hkv * T_cap + kept * 4 + B * Hkv * 8


def repack_bytes(n2, n1, D, G):
    """Per kept token: bf16 K and V read, its position, codes + (scale, zero) written."""
    r6, r4, sz = D * 6 // 8, D * 4 // 8, sz_bytes(D, G)
    return (n2 + n1) * (2 * D * 2 + 4 + r6 + sz) + n2 * (r6 + sz) + n1 * (r4 + sz)


def tiered_bytes(n2, n1, skipped_rows, B, Hq, Hkv, D, G):
    """K rows of the kept tokens, their V rows unless every head skips them, q, out, the counts."""
    r6, r4, sz = D * 6 // 8, D * 4 // 8, sz_bytes(D, G)
    kept = n2 + n1
    v_kept = n2 * (r6 + sz) + n1 * (r4 + sz)
    keep_frac = 1.0 - skipped_rows / kept if kept else 0.0
    return kept * (r6 + sz) + int(round(v_kept * keep_frac)) + B * Hq * D * 6 + B * Hkv * 8


def path_bytes(cfg, seq_lens, counts, skipped_rows, skipped_rows_tiered):
    """Algorithmic HBM bytes of each kernel of one step of the main workload."""
    D, G, Hkv, Hq = cfg.D, cfg.G, cfg.Hkv, cfg.Hq
    B, T_cap = len(seq_lens), cfg.T_cap
    rows = int(np.asarray(seq_lens, np.int64).sum()) * Hkv
    n2, n1 = int(np.asarray(counts)[..., 0].sum()), int(np.asarray(counts)[..., 1].sum())
    return {
        "quantize": quantize_bytes(rows, D, G, KB, VB),
        "decode": decode_bytes(rows, rows - skipped_rows, B, Hq, D, G, KB, VB),
        "classify": classify_bytes(rows, B, Hkv, T_cap, n2 + n1),
        "repack": repack_bytes(n2, n1, D, G),
        "tiered": tiered_bytes(n2, n1, skipped_rows_tiered, B, Hq, Hkv, D, G),
    }


# ----------------------------------------------------------------- ranks and timing

def rank_workload(rank):
    """The batch rank `rank` decodes: the main workload with its own seed, so
    the ranks process distinct, independent batches (weak scaling)."""
    base = W.CONFIGS[CFG_MAIN]
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


def job_throughput(bytes_per_rank, world, seconds):
    """Whole-job GB/s: the bytes all ranks moved over the slowest rank's time."""
    return bytes_per_rank * world / seconds / 1e9


class Timed:
    """Runs named launches in order, steps times, with L2 flushed before each
    launch outside its event pair; keeps every launch's device time (ms)."""

    def __init__(self, device, stream):
        self.stream = stream
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def run(self, launches, steps, warmup, on_step=None):
        for _ in range(warmup):
            for _, fn in launches:
                self.flush.zero_()
                fn()
        torch.cuda.synchronize()
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in launches] for _ in range(steps)]
        for i in range(steps):
            for j, (_, fn) in enumerate(launches):
                self.flush.zero_()
                ev[i][j][0].record(self.stream)
                fn()
                ev[i][j][1].record(self.stream)
            if on_step is not None:
                on_step(i)
        torch.cuda.synchronize()
        return {name: [ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(steps)]
                for j, (name, _) in enumerate(launches)}


def launch_floor_us(timer, steps):
    """Device time of a trivial kernel (zeroing 4 KB) timed exactly like the
    library's kernels: the floor under every small launch of this harness."""
    small = torch.empty(1024, device=timer.flush.device)
    t = timer.run([("floor", lambda: small.zero_())], max(steps, 10), 3)
    return round(statistics.median(t["floor"]) * 1e3, 2)


def kernel_line(ms_list, nbytes, peak):
    ms = statistics.median(ms_list)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"us": round(ms * 1e3, 2), "bytes": int(nbytes), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}


# ----------------------------------------------------------------- the main step

class Step:
    """Device buffers and the five launches of one step of the main workload."""

    def __init__(self, cfg, inp, device):
        from quantized_kv_cache_lkv_b200 import buffers, lkv
        self.lkv = lkv
        self.cfg = cfg
        B, Hq, Hkv, D, T, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.G
        self.shape = (B, Hq, Hkv, D, T, G)
        self.d = {k: v.to(device) for k, v in inp.items()}
        self.cache = buffers.alloc_cache(KB, VB, G, B, Hkv, T, D, device, zero=True)
        self.out = torch.empty(B, Hq, D, device=device)
        self.out2 = torch.empty(B, Hq, D, device=device)
        self.cnt = torch.zeros(2, dtype=torch.int64, device=device)
        self.cnt2 = torch.zeros(2, dtype=torch.int64, device=device)
        self.ws = buffers.alloc_workspace(lkv.lkv_decode_workspace_bytes((KB, VB, G), B, Hq, Hkv, T, D), device)
        self.ws2 = buffers.alloc_workspace(lkv.lkv_tiered_workspace_bytes(B, Hq, Hkv, T, D, G), device)
        self.tiers = buffers.alloc_tiers(B, Hkv, T, device, zero=True)
        self.A, self.Bs = buffers.alloc_segments(G, B, Hkv, T, D, device, zero=True)

    def quantize(self, s=None):
        B, Hq, Hkv, D, T, G = self.shape
        d, c = self.d, self.cache
        self.lkv.lkv_quantize_kv((KB, VB, G), B, Hkv, T, D, d["seq_lens"], d["k"], d["v"], c["k_codes"],
                                 c["k_sz"], c["v_codes"], c["v_sz"], s)

    def decode(self, s=None, seq_lens=None, q=None):
        B, Hq, Hkv, D, T, G = self.shape
        d, c = self.d, self.cache
        self.lkv.lkv_decode_attention((KB, VB, G), B, Hq, Hkv, T, D,
                                      d["seq_lens"] if seq_lens is None else seq_lens,
                                      d["q"] if q is None else q, c["k_codes"], c["k_sz"], c["v_codes"],
                                      c["v_sz"], self.cfg.softmax_scale, self.cfg.tau, self.out, None, self.cnt,
                                      self.ws, self.ws.numel(), s)

    def classify(self, s=None):
        B, Hq, Hkv, D, T, G = self.shape
        t, d = self.tiers, self.d
        self.lkv.lkv_tier_classify(B, Hkv, T, d["seq_lens"], d["mass"], TAU_LOW, TAU_HIGH, t["tier"],
                                   t["counts"], t["pos_a"], t["pos_b"], s)

    def repack(self, s=None):
        B, Hq, Hkv, D, T, G = self.shape
        t, d = self.tiers, self.d
        self.lkv.lkv_tier_repack(B, Hkv, T, D, G, d["k"], d["v"], t["counts"], t["pos_a"], t["pos_b"], self.A,
                                 self.Bs, s)

    def tiered(self, s=None):
        B, Hq, Hkv, D, T, G = self.shape
        self.lkv.lkv_tiered_attention(B, Hq, Hkv, T, D, G, self.tiers["counts"], self.d["q"], self.A, self.Bs,
                                      self.cfg.softmax_scale, 0.0, self.out2, self.cnt2, self.ws2,
                                      self.ws2.numel(), s)

    def launches(self, stream):
        s = stream.cuda_stream
        return [("quantize", lambda: self.quantize(s)), ("decode", lambda: self.decode(s)),
                ("classify", lambda: self.classify(s)), ("repack", lambda: self.repack(s)),
                ("tiered", lambda: self.tiered(s))]

    LAUNCHES_PER_STEP = 5    # quantize, decode, classify, repack, tiered: one kernel each

    def algorithmic_bytes(self):
        """Bytes each kernel must move, from the step's device results."""
        sl = self.d["seq_lens"].cpu().numpy()
        counts = self.tiers["counts"].cpu().numpy()
        self.skipped_rows = int(self.cnt[1].item())
        by = path_bytes(self.cfg, sl, counts, self.skipped_rows, int(self.cnt2[1].item()))
        self.kept = (int(counts[..., 0].sum()), int(counts[..., 1].sum()),
                     int(sl.astype(np.int64).sum()) * self.cfg.Hkv)
        return by


def run_e2e(step, inp, device, stream, steps):
    """Decode loop through the public API with host buffers.  The cache holds
    the workload's tokens; the loop starts `steps` tokens short of the full
    context and, every step, copies that step's inputs (q, the new token's
    K/V, its position and the new lengths, packed in one pinned staging
    buffer) host->device in one copy, appends the token (lkv_append_kv),
    decodes over the longer sequences, and copies out and the skip counts
    (adjacent in one device buffer) back in one copy."""
    cfg = step.cfg
    B, Hq, Hkv, D, T, G = step.shape
    L = step.lkv
    s = stream.cuda_stream
    full = inp["seq_lens"].to(torch.int64)
    start = torch.clamp(full - steps, min=0)
    pos = torch.stack([torch.clamp(start + i, max=T - 1) for i in range(steps)]).to(torch.int32)
    lens = torch.stack([torch.minimum(start + i + 1, full) for i in range(steps)]).to(torch.int32)
    idx = pos.to(torch.int64)
    # staging layout per step (every part a multiple of 16 bytes): q | k | v | pos | lens
    nq, nkv = B * Hq * D * 2, B * Hkv * D * 2
    parts = [nq, nkv, nkv, B * 4, B * 4]
    offs = [sum(parts[:i]) for i in range(len(parts))]
    per_step = (sum(parts) + 255) // 256 * 256
    h_in = torch.empty(steps, per_step, dtype=torch.uint8).pin_memory()
    for i in range(steps):
        row = h_in[i]
        row[offs[0]:offs[0] + nq].copy_(inp["q"].contiguous().view(-1).view(torch.uint8))
        row[offs[1]:offs[1] + nkv].copy_(inp["k"][torch.arange(B), :, idx[i]].contiguous().view(-1).view(torch.uint8))
        row[offs[2]:offs[2] + nkv].copy_(inp["v"][torch.arange(B), :, idx[i]].contiguous().view(-1).view(torch.uint8))
        row[offs[3]:offs[3] + B * 4].copy_(pos[i].view(torch.uint8))
        row[offs[4]:offs[4] + B * 4].copy_(lens[i].view(torch.uint8))
    d_in = torch.empty(per_step, dtype=torch.uint8, device=device)
    d_q = d_in[offs[0]:offs[0] + nq].view(torch.bfloat16).view(B, Hq, D)
    d_k = d_in[offs[1]:offs[1] + nkv].view(torch.bfloat16).view(B, Hkv, D)
    d_v = d_in[offs[2]:offs[2] + nkv].view(torch.bfloat16).view(B, Hkv, D)
    d_pos = d_in[offs[3]:offs[3] + B * 4].view(torch.int32)
    d_len = d_in[offs[4]:offs[4] + B * 4].view(torch.int32)
    n_out = B * Hq * D * 4
    d_res = torch.empty(n_out + 16, dtype=torch.uint8, device=device)   # out (f32) then the two skip counts
    out = d_res[:n_out].view(torch.float32).view(B, Hq, D)
    cnt = d_res[n_out:].view(torch.int64)
    h_res = torch.empty(steps, n_out + 16, dtype=torch.uint8).pin_memory()
    c = step.cache

    def one(i):
        d_in.copy_(h_in[i], non_blocking=True)
        L.lkv_append_kv((KB, VB, G), B, Hkv, T, D, d_pos, d_k, d_v, c["k_codes"], c["k_sz"], c["v_codes"],
                        c["v_sz"], s)
        L.lkv_decode_attention((KB, VB, G), B, Hq, Hkv, T, D, d_len, d_q, c["k_codes"], c["k_sz"],
                               c["v_codes"], c["v_sz"], cfg.softmax_scale, cfg.tau, out, None, cnt, step.ws,
                               step.ws.numel(), s)
        h_res[i].copy_(d_res, non_blocking=True)

    one(0)                                   # warm-up (rewrites the same row)
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        one(i)
    t1.record(stream)
    torch.cuda.synchronize(device)
    sec = t0.elapsed_time(t1) * 1e-3
    by = 0
    for i in range(steps):
        rows = int(lens[i].to(torch.int64).sum()) * Hkv
        skipped = int(h_res[i, n_out:].view(torch.int64)[1])
        by += decode_bytes(rows, rows - skipped, B, Hq, D, G, KB, VB)
        by += quantize_bytes(B * Hkv, D, G, KB, VB)           # the appended rows
    return {"value": round(by / sec / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": int(sum(parts)),
            "d2h_bytes_per_step": int(n_out + 16), "seconds": sec, "bytes": by, "steps": steps,
            "us_per_step": round(sec / steps * 1e6, 2),
            "loop": "one H2D copy of q + new K/V + pos + lengths, lkv_append_kv, lkv_decode_attention, "
                    "one D2H copy of out + skip counts"}


def bench_stream(step, device, stream, args, peak, nbytes, copies=4, blocks=5):
    """The decode call back to back over `copies` copies of the cache (the
    step's quantized cache plus copies), one event pair per block of calls."""
    caches = [step.cache] + [{k: t.clone() for k, t in step.cache.items()} for _ in range(copies - 1)]
    B, Hq, Hkv, D, T, G = step.shape
    L, s, cfg, d = step.lkv, stream.cuda_stream, step.cfg, step.d

    def call(c):
        L.lkv_decode_attention((KB, VB, G), B, Hq, Hkv, T, D, d["seq_lens"], d["q"], c["k_codes"], c["k_sz"],
                               c["v_codes"], c["v_sz"], cfg.softmax_scale, cfg.tau, step.out, None, step.cnt,
                               step.ws, step.ws.numel(), s)

    per_block = max(args.steps, 4 * copies) // copies * copies
    for i in range(2 * copies):
        call(caches[i % copies])
    torch.cuda.synchronize(device)
    ms = []
    for _ in range(blocks):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(per_block):
            call(caches[i % copies])
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms.append(e0.elapsed_time(e1) / per_block)
    line = kernel_line(ms, nbytes, peak)
    line.update({"calls_per_block": per_block, "blocks": blocks, "cache_copies": copies,
                 "l2": f"inputs larger than L2: {copies} cache copies of "
                       f"{sum(t.numel() * t.element_size() for t in step.cache.values()) >> 20} MiB rotated, no flush"})
    del caches
    torch.cuda.empty_cache()
    return line


def run_one_call(args, step, timer, stream):
    """--call: one untimed pass of the whole step, then only the named call,
    warm-up + timed steps with L2 flushed before each; prints its median."""
    launches = dict(step.launches(stream))
    for fn in launches.values():
        fn()
    t = timer.run([(args.call, launches[args.call])], args.steps, args.warmup)
    print(json.dumps({"call": args.call, "workload": step.cfg.name, "steps": args.steps,
                      "us_median": round(statistics.median(t[args.call]) * 1e3, 2)}), flush=True)


# ----------------------------------------------------------------- other workloads (1 GPU)

def bench_long(device, stream, timer, args, peak):
    from quantized_kv_cache_lkv_b200 import buffers, lkv
    cfg = W.CONFIGS[CFG_LONG]
    B, Hq, Hkv, D, T, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.G
    inp = {k: v.to(device) for k, v in W.make_inputs(cfg).items()}
    cache = buffers.alloc_cache(KB, VB, G, B, Hkv, T, D, device, zero=True)
    out = torch.empty(B, Hq, D, device=device)
    cnt = torch.zeros(2, dtype=torch.int64, device=device)
    ws = buffers.alloc_workspace(lkv.lkv_decode_workspace_bytes((KB, VB, G), B, Hq, Hkv, T, D), device)
    s = stream.cuda_stream
    quant = lambda: lkv.lkv_quantize_kv((KB, VB, G), B, Hkv, T, D, inp["seq_lens"], inp["k"], inp["v"],
                                        cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"], s)
    dec = lambda: lkv.lkv_decode_attention((KB, VB, G), B, Hq, Hkv, T, D, inp["seq_lens"], inp["q"],
                                           cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"],
                                           cfg.softmax_scale, cfg.tau, out, None, cnt, ws, ws.numel(), s)
    t = timer.run([("quantize", quant), ("decode", dec)], args.steps, args.warmup)
    rows = int(inp["seq_lens"].sum()) * Hkv
    skipped = int(cnt[1].item())
    dline = kernel_line(t["decode"], decode_bytes(rows, rows - skipped, B, Hq, D, G, KB, VB), peak)
    dline["v_rows_skipped_frac"] = round(skipped / rows, 4)
    dline["kv_tokens_per_s"] = round(rows / Hkv / (dline["us"] * 1e-6), 1)
    res = {"workload": cfg.name, "decode": dline,
           "quantize": kernel_line(t["quantize"], quantize_bytes(rows, D, G, KB, VB), peak)}
    del inp, cache, ws
    torch.cuda.empty_cache()
    return res


def fp64_reference(inp, cfg):
    """fp64 softmax attention over the unquantized bf16 K/V, with torch on the
    device (the quality yardstick of the bit-width sweep)."""
    B, Hq, Hkv, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.D
    r = Hq // Hkv
    out = torch.zeros(B, Hq, D, dtype=torch.float64, device=inp["q"].device)
    for b in range(B):
        T = int(inp["seq_lens"][b])
        if T == 0:
            continue
        K = inp["k"][b, :, :T].double()                                  # [Hkv, T, D]
        V = inp["v"][b, :, :T].double()
        q = inp["q"][b].double().view(Hkv, r, D)
        s = torch.einsum("grd,gtd->grt", q, K) * cfg.softmax_scale
        out[b] = torch.einsum("grt,gtd->grd", torch.softmax(s, dim=-1), V).reshape(Hq, D)
    return out


def bench_sweep(device, stream, timer, args, peak):
    from quantized_kv_cache_lkv_b200 import buffers, lkv
    cfg = W.CONFIGS[CFG_SWEEP]
    B, Hq, Hkv, D, T, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.G
    inp = {k: v.to(device) for k, v in W.make_inputs(cfg).items()}
    ref = fp64_reference(inp, cfg)
    rows = int(inp["seq_lens"].sum()) * Hkv
    out = torch.empty(B, Hq, D, device=device)
    cnt = torch.zeros(2, dtype=torch.int64, device=device)
    s = stream.cuda_stream
    res = {"workload": cfg.name}
    for kb, vb in cfg.bits:
        cache = buffers.alloc_cache(kb, vb, G, B, Hkv, T, D, device, zero=True)
        ws = buffers.alloc_workspace(lkv.lkv_decode_workspace_bytes((kb, vb, G), B, Hq, Hkv, T, D), device)
        lkv.lkv_quantize_kv((kb, vb, G), B, Hkv, T, D, inp["seq_lens"], inp["k"], inp["v"], cache["k_codes"],
                            cache["k_sz"], cache["v_codes"], cache["v_sz"], s)
        dec = (lambda kb=kb, vb=vb, cache=cache, ws=ws: lkv.lkv_decode_attention(
            (kb, vb, G), B, Hq, Hkv, T, D, inp["seq_lens"], inp["q"], cache["k_codes"], cache["k_sz"],
            cache["v_codes"], cache["v_sz"], cfg.softmax_scale, cfg.tau, out, None, cnt, ws, ws.numel(), s))
        t = timer.run([("decode", dec)], args.steps, args.warmup)
        skipped = int(cnt[1].item())
        line = kernel_line(t["decode"], decode_bytes(rows, rows - skipped, B, Hq, D, G, kb, vb), peak)
        # compression: bytes the buffers give one valid row, against bf16 K + V
        row_q = (cache["k_codes"].shape[-1] + cache["v_codes"].shape[-1]
                 + (cache["k_sz"][0, 0, 0].numel() + cache["v_sz"][0, 0, 0].numel()) * 4)
        formula = (2 * 16 * D) / ((kb + vb) * D + 2 * 64 * (D // G))
        err = (out.double() - ref).norm() / ref.norm()
        line.update({"compression": {"measured": round(2 * D * 2 / row_q, 4), "formula": round(formula, 4)},
                     "rel_l2_vs_bf16_fp64": float(f"{err.item():.4e}")})
        res[f"K{kb}V{vb}"] = line
        del cache, ws
    del inp, ref
    torch.cuda.empty_cache()
    return res


def bench_tiered(device, stream, timer, args, peak):
    from quantized_kv_cache_lkv_b200 import buffers, lkv
    cfg = W.CONFIGS[CFG_TIER]
    B, Hq, Hkv, D, T, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.G
    inp = {k: v.to(device) for k, v in W.make_inputs(cfg, with_mass=True).items()}
    tiers = buffers.alloc_tiers(B, Hkv, T, device, zero=True)
    A, Bs = buffers.alloc_segments(G, B, Hkv, T, D, device, zero=True)
    out = torch.empty(B, Hq, D, device=device)
    cnt = torch.zeros(2, dtype=torch.int64, device=device)
    ws = buffers.alloc_workspace(lkv.lkv_tiered_workspace_bytes(B, Hq, Hkv, T, D, G), device)
    s = stream.cuda_stream
    lo, hi = cfg.tau_low, cfg.tau_high
    launches = [
        ("classify", lambda: lkv.lkv_tier_classify(B, Hkv, T, inp["seq_lens"], inp["mass"], lo, hi, tiers["tier"],
                                                   tiers["counts"], tiers["pos_a"], tiers["pos_b"], s)),
        ("repack", lambda: lkv.lkv_tier_repack(B, Hkv, T, D, G, inp["k"], inp["v"], tiers["counts"],
                                               tiers["pos_a"], tiers["pos_b"], A, Bs, s)),
        ("tiered", lambda: lkv.lkv_tiered_attention(B, Hq, Hkv, T, D, G, tiers["counts"], inp["q"], A, Bs,
                                                    cfg.softmax_scale, cfg.tau, out, cnt, ws, ws.numel(), s)),
    ]
    t = timer.run(launches, args.steps, args.warmup)
    counts = tiers["counts"].cpu().numpy()
    n2, n1 = int(counts[..., 0].sum()), int(counts[..., 1].sum())
    rows = int(inp["seq_lens"].sum()) * Hkv
    r6, r4, sz = D * 6 // 8, D * 4 // 8, sz_bytes(D, G)
    tiered_cache = n2 * (2 * r6 + 2 * sz) + n1 * (r6 + r4 + 2 * sz)
    k6v4_cache = rows * (r6 + r4 + 2 * sz)
    res = {
        "workload": cfg.name,
        "classify": kernel_line(t["classify"], classify_bytes(rows, B, Hkv, T, n2 + n1), peak),
        "repack": kernel_line(t["repack"], repack_bytes(n2, n1, D, G), peak),
        "tiered_decode": kernel_line(t["tiered"], tiered_bytes(n2, n1, int(cnt[1].item()), B, Hq, Hkv, D, G), peak),
        "tiers": {"v6": n2, "v4": n1, "evicted": rows - n2 - n1, "rows": rows},
        "compression": {"vs_bf16": round(rows * 2 * D * 2 / max(tiered_cache, 1), 3),
                        "vs_k6v4_cache": round(k6v4_cache / max(tiered_cache, 1), 3)},
    }
    del inp, tiers, A, Bs, ws
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------- the GPU arm

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
    timer = Timed(device, stream)
    peak, peak_kind = peaks()

    def barrier():
        if dist:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)

    if args.call:
        run_one_call(args, step, timer, stream)
        return

    launches = step.launches(stream)
    for _ in range(args.warmup):
        for _, fn in launches:
            timer.flush.zero_()
            fn()
    barrier()
    with ClockSampler(local) as clocks:
        barrier()
        times = timer.run(launches, args.steps, 0)
        barrier()
    by = step.algorithmic_bytes()
    dec_ms = max_over_ranks(statistics.median(times["decode"]), device)
    value = job_throughput(by["decode"], world, dec_ms * 1e-3)
    step_ms_list = [sum(times[n][i] for n, _ in launches) for i in range(args.steps)]
    step_ms = max_over_ranks(statistics.median(step_ms_list), device)
    kern = {}
    for name, _ in launches:
        kern[name] = kernel_line(times[name], by[name], peak)
        kern[name]["share"] = round(statistics.median(times[name]) / statistics.median(step_ms_list), 4)
    traffic = traffic_table()

    def roofline(name):
        tr = traffic.get(name)
        t_bytes = tr[1] if tr and tr[0] == source_hash(name) else None
        return {"bound": "hbm", "achieved": kern[name]["gbs"], "peak": peak, "unit": "GB/s",
                "frac": kern[name]["frac"], "traffic": t_bytes, "kernel": name,
                "algorithmic_bytes": by[name], "peak_source": f"{peak_kind} hbm_gbs (of {peak_kind})"}

    e2e = None
    if not args.no_e2e:   # every rank runs it; the job's time is the slowest rank's
        e2e = run_e2e(step, inp, device, stream, max(args.steps, 20))
        sec = max_over_ranks(e2e["seconds"], device)
        e2e["value"] = round(job_throughput(e2e["bytes"], world, sec), 2)
    extras = {"launch_floor_us": launch_floor_us(timer, args.steps)}
    if world == 1 and not args.no_extras:
        extras["stream"] = bench_stream(step, device, stream, args, peak, by["decode"])
        extras["stream"]["kv_tokens_per_s"] = round(step.kept[2] / cfg.Hkv / (extras["stream"]["us"] * 1e-6), 1)
    if world == 1 and not args.no_extras:
        del step.d["k"], step.d["v"]
        torch.cuda.empty_cache()
        extras["long_context"] = bench_long(device, stream, timer, args, peak)
        extras["bit_sweep"] = bench_sweep(device, stream, timer, args, peak)
        extras["tiered"] = bench_tiered(device, stream, timer, args, peak)
    cpu = cpu_baseline(cfg, inp, args) if rank == 0 and world == 1 and not args.no_cpu else None

    if rank == 0:
        clk = clocks.summary()
        rows = step.kept[2]
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dec_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "head_dim": cfg.D,
                       "context": cfg.T_cap, "group": cfg.G, "k_bits": KB, "v_bits": VB, "tau": cfg.tau,
                       "heavy_hitters": cfg.hh_frac,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "value": "lkv_decode_attention algorithmic GB/s, median over the timed steps",
                       "l2": "flushed (512 MiB write) before every kernel, outside its events"},
            "kv_tokens_per_s": round(rows / cfg.Hkv * world / (dec_ms * 1e-3), 1),
            "roofline": roofline("decode"),
            "decode_skip": {"v_rows_skipped": step.skipped_rows, "rows": rows,
                            "frac": round(step.skipped_rows / max(rows, 1), 4),
                            "dense_bytes": decode_bytes(rows, rows, cfg.B, cfg.Hq, cfg.D, cfg.G, KB, VB)},
            "step": {"ms": round(step_ms, 5), "gbs": round(job_throughput(sum(by.values()), world, step_ms * 1e-3), 1),
                     "kernels": kern, "dominant_roofline": roofline(max(kern, key=lambda k: kern[k]["us"])),
                     "tiers": {"v6": step.kept[0], "v4": step.kept[1], "rows": rows,
                               "tau_low": TAU_LOW, "tau_high": TAU_HIGH},
                     "what": "quantize + decode + tier classify + repack + tiered decode"},
            "gpu_launches": Step.LAUNCHES_PER_STEP * args.steps,
            "clocks": {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "e2e": {k: e2e[k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step",
                                        "us_per_step", "steps", "loop")} if e2e else None,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ----------------------------------------------------------------- CPU oracle

def oracle_decode_gbs(orc, cfg, sub, passes_seconds):
    """The oracle's decode over a sample, repeated for about passes_seconds:
    (GB/s of the decode metric, passes, seconds)."""
    k, v, q = W.bf16_bits(sub["k"]), W.bf16_bits(sub["v"]), W.bf16_bits(sub["q"])
    sl = sub["seq_lens"].numpy()
    cache = orc.quantize_kv(KB, VB, cfg.G, k, v, sl)
    rows = int(sl.astype(np.int64).sum()) * cfg.Hkv
    total_by, total_dt, passes = 0, 0.0, 0
    while total_dt < passes_seconds or passes == 0:
        t0 = time.perf_counter()
        _, _, cnt = orc.decode_attention(KB, VB, cfg.G, sl, q, cache, cfg.softmax_scale, cfg.tau, want_mask=False)
        total_dt += time.perf_counter() - t0
        total_by += decode_bytes(rows, rows - int(cnt[1]), len(sl), cfg.Hq, cfg.D, cfg.G, KB, VB)
        passes += 1
    return total_by / total_dt / 1e9, passes, total_dt


def oracle_sample(cfg, inp, n_seq):
    return {k: inp[k][:n_seq].contiguous() for k in ("q", "k", "v", "seq_lens", "mass")}


def cpu_baseline(cfg, inp, args):
    """The oracle's decode on the host cores (all of them, then one), on
    samples of the main workload sized to about --cpu-seconds each."""
    import oracle
    oracle.lib()
    all_cores = oracle.threads()
    gbs, passes, dt = oracle_decode_gbs(oracle, cfg, oracle_sample(cfg, inp, cfg.B), args.cpu_seconds)
    oracle.set_threads(1)
    n1 = 1
    gbs1, passes1, dt1 = oracle_decode_gbs(oracle, cfg, oracle_sample(cfg, inp, n1), args.cpu_seconds)
    oracle.set_threads(all_cores)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": all_cores, "kind": "oracle",
            "sample": f"all {cfg.B} sequences of {cfg.name}, oracle decode (fp64), {passes} pass(es) in {dt:.1f} s",
            "one_thread": {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                           "sample": f"first {n1} of {cfg.B} sequences, {passes1} pass(es) in {dt1:.1f} s"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.lib()
    cfg = W.CONFIGS[CFG_MAIN]
    inp = W.make_inputs(cfg, with_mass=True)
    k, v, q = W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"]), W.bf16_bits(inp["q"])
    sl = inp["seq_lens"].numpy()
    cache = oracle.quantize_kv(KB, VB, cfg.G, k, v, sl)
    rows = int(sl.astype(np.int64).sum()) * cfg.Hkv
    times, by = [], 0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        _, _, cnt = oracle.decode_attention(KB, VB, cfg.G, sl, q, cache, cfg.softmax_scale, cfg.tau,
                                            want_mask=False)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            by = decode_bytes(rows, rows - int(cnt[1]), cfg.B, cfg.Hq, cfg.D, cfg.G, KB, VB)
    med = statistics.median(times)
    value = by / med / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(med * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "head_dim": cfg.D,
                   "context": cfg.T_cap, "group": cfg.G, "k_bits": KB, "v_bits": VB, "tau": cfg.tau,
                   "parallelism": "single",
                   "value": "oracle decode algorithmic GB/s, median over the timed steps"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"all {cfg.B} sequences per step, oracle decode (fp64)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lkv", "reference"], default="lkv")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    ap.add_argument("--no-extras", action="store_true", help="skip the long-context, sweep and tiered workloads")
    ap.add_argument("--call", choices=["quantize", "decode", "classify", "repack", "tiered"],
                    help="time only this call of the step (for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_lkv(args)


if __name__ == "__main__":
    main()
