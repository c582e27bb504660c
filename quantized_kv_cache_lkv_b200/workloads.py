"""Seeded synthetic workloads for the quantized-KV decode path.

This module only draws random inputs; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Shapes follow the Llama-3.1-8B KV geometry the Super KV Compression page
quotes its K6V4 results on (32 query heads, 8 KV heads, head_dim 128); the
pages publish no dataset for the kernel itself, so every input is synthetic:

* K ~ N(0, 1) * s[hkv, d], with s log-uniform in [0.5, 4] per (KV head,
  channel) and two outlier channels per KV head scaled by 15 more;
* V ~ N(0, 1), q ~ N(0, 1);
* heavy hitters: round(f * T_b) positions per sequence (shared by the KV
  heads) whose K row is 4 * mean(q of the group) + N(0, 1), which makes the
  softmax peaky;
* previous-step attention mass (tiered cache): a_t = r_t^-1.1 / sum_r r^-1.1
  with r a random permutation of 1..T_b per (sequence, KV head) -- a Zipf(1.1)
  law over token positions.

Values are drawn in fp32 and rounded to bf16 (round to nearest even).
Positions t >= T_b of the [B, Hkv, T_cap, D] cache tensors are zero.
"""
from dataclasses import dataclass, field
import math
from typing import List, Optional, Tuple

import torch


@dataclass
class Config:
    """One workload: shapes, quantizer, skip threshold and input recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    T_cap: int
    G: int
    bits: List[Tuple[int, int]]          # (k_bits, v_bits) settings to run
    tau: float = 0.0                     # sparse-V skip threshold
    hh_frac: float = 0.0                 # heavy-hitter fraction per sequence
    seq: str = "fixed"                   # fixed | uniform | loguniform
    seq_lo: int = 0
    seq_hi: int = 0
    tau_low: Optional[float] = None      # tier thresholds (tiered cache only)
    tau_high: Optional[float] = None
    seed: int = 0
    note: str = ""

    @property
    def r(self):
        return self.Hq // self.Hkv

    @property
    def softmax_scale(self):
        return float(torch.tensor(1.0 / math.sqrt(self.D), dtype=torch.float32))


CONFIGS = {
    1: Config("tiny_k6v4", B=1, Hq=4, Hkv=2, D=64, T_cap=256, G=32, bits=[(6, 4)], tau=0.0,
              seed=0, note="batch 1, 4q/2kv heads, head_dim 64, context 256, group 32"),
    2: Config("llama8b_k6v4_b16_t8192", B=16, Hq=32, Hkv=8, D=128, T_cap=8192, G=64,
              bits=[(6, 4)], tau=1e-4, hh_frac=0.01, seed=1,
              note="Llama-3.1-8B-shaped single layer decode, 1% heavy hitters, tau 1e-4"),
    3: Config("long_k6v4_b1_t131072", B=1, Hq=32, Hkv=8, D=128, T_cap=131072, G=64,
              bits=[(6, 4)], tau=1e-5, hh_frac=0.001, seed=2,
              note="long context, 0.1% heavy hitters, tau 1e-5"),
    4: Config("sweep_ragged_b64", B=64, Hq=32, Hkv=8, D=128, T_cap=4096, G=32,
              bits=[(8, 8), (6, 4), (4, 4), (4, 2)], tau=0.0, seq="uniform",
              seq_lo=512, seq_hi=4096, seed=3,
              note="bit-width sweep, ragged context uniform in [512, 4096]"),
    5: Config("tiered_b32", B=32, Hq=32, Hkv=8, D=128, T_cap=32768, G=64, bits=[(6, 6), (6, 4)],
              tau=0.0, seq="loguniform", seq_lo=1024, seq_hi=32768, tau_low=1e-4,
              tau_high=1e-2, seed=4,
              note="attention-tiered cache, context log-uniform in [1024, 32768], Zipf(1.1) mass"),
}


def scaled(cfg: Config, **kw) -> Config:
    """A copy of cfg with some fields replaced (smaller parity cases)."""
    d = dict(cfg.__dict__)
    d.update(kw)
    return Config(**d)


def seq_lens_for(cfg: Config, gen: torch.Generator) -> torch.Tensor:
    if cfg.seq == "fixed":
        return torch.full((cfg.B,), cfg.T_cap, dtype=torch.int32)
    if cfg.seq == "uniform":
        return torch.randint(cfg.seq_lo, cfg.seq_hi + 1, (cfg.B,), generator=gen,
                             dtype=torch.int64).to(torch.int32)
    if cfg.seq == "loguniform":
        u = torch.rand(cfg.B, generator=gen, dtype=torch.float64)
        t = torch.exp(math.log(cfg.seq_lo) + u * (math.log(cfg.seq_hi) - math.log(cfg.seq_lo)))
        return torch.clamp(torch.floor(t), cfg.seq_lo, cfg.seq_hi).to(torch.int32)
    raise ValueError(cfg.seq)


def make_inputs(cfg: Config, seq_lens: Optional[torch.Tensor] = None, with_mass: bool = False):
    """Draw (q, k, v, seq_lens[, mass]) on the CPU from cfg.seed.

    q: bf16 [B, Hq, D]; k, v: bf16 [B, Hkv, T_cap, D]; seq_lens: int32 [B];
    mass: f32 [B, Hkv, T_cap] (zero beyond T_b).
    """
    gen = torch.Generator().manual_seed(cfg.seed)
    B, Hq, Hkv, D, T_cap, r = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.r
    if seq_lens is None:
        seq_lens = seq_lens_for(cfg, gen)
    seq_lens = seq_lens.to(torch.int32)
    # per-(KV head, channel) K scale, log-uniform in [0.5, 4], two outliers x15
    u = torch.rand(Hkv, D, generator=gen, dtype=torch.float32)
    s = torch.exp(math.log(0.5) + u * (math.log(4.0) - math.log(0.5)))
    for g in range(Hkv):
        ch = torch.randperm(D, generator=gen)[:2]
        s[g, ch] *= 15.0
    q32 = torch.randn(B, Hq, D, generator=gen, dtype=torch.float32)
    q = q32.to(torch.bfloat16)
    k = torch.zeros(B, Hkv, T_cap, D, dtype=torch.bfloat16)
    v = torch.zeros(B, Hkv, T_cap, D, dtype=torch.bfloat16)
    for b in range(B):
        T = int(seq_lens[b])
        if T <= 0:
            continue
        kb = torch.randn(Hkv, T, D, generator=gen, dtype=torch.float32) * s[:, None, :]
        n_hh = int(round(cfg.hh_frac * T))
        if n_hh > 0:
            pos = torch.randperm(T, generator=gen)[:n_hh]
            qbar = q[b].float().view(Hkv, r, D).mean(dim=1)                 # [Hkv, D]
            noise = torch.randn(Hkv, n_hh, D, generator=gen, dtype=torch.float32)
            kb[:, pos, :] = 4.0 * qbar[:, None, :] + noise
        k[b, :, :T] = kb.to(torch.bfloat16)
        v[b, :, :T] = torch.randn(Hkv, T, D, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    out = {"q": q, "k": k, "v": v, "seq_lens": seq_lens}
    if with_mass:
        out["mass"] = make_mass(cfg, seq_lens, gen)
    return out


def make_mass(cfg: Config, seq_lens: torch.Tensor, gen: torch.Generator, s: float = 1.1):
    """Zipf(s) attention mass over a random ranking of each sequence's tokens."""
    mass = torch.zeros(cfg.B, cfg.Hkv, cfg.T_cap, dtype=torch.float32)
    for b in range(cfg.B):
        T = int(seq_lens[b])
        if T <= 0:
            continue
        ranks = torch.arange(1, T + 1, dtype=torch.float64)
        w = ranks.pow(-s)
        w = w / w.sum()
        for g in range(cfg.Hkv):
            perm = torch.randperm(T, generator=gen)
            mass[b, g, :T] = w[perm].to(torch.float32)
    return mass


def bf16_bits(t: torch.Tensor):
    """Raw uint16 bits of a CPU bf16 tensor as a numpy array."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
