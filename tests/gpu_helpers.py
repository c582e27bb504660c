"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the CPU oracle on the same seeded inputs."""
import numpy as np
import torch

from quantized_kv_cache_lkv_b200 import buffers, lkv
from quantized_kv_cache_lkv_b200 import workloads as W

# Tolerances of the attention outputs (fp32 path vs fp64 oracle).
REL_L2 = 1e-5
MAX_ABS_PER_VMAX = 5e-5
TIE_BAND = 1e-7   # |p - tau| below this may fall either side of the skip test


def dev(t):
    return t.to("cuda", non_blocking=False).contiguous()


def gpu_quantize(kb, vb, G, inp, zero=True):
    q = inp
    B, Hkv, T_cap, D = q["k"].shape
    cache = buffers.alloc_cache(kb, vb, G, B, Hkv, T_cap, D, zero=zero)
    lkv.lkv_quantize_kv((kb, vb, G), B, Hkv, T_cap, D, dev(q["seq_lens"]), dev(q["k"]), dev(q["v"]),
                        cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"])
    torch.cuda.synchronize()
    return cache


def gpu_decode(kb, vb, G, inp, cache, softmax_scale, tau, want_mask=True, ws=None):
    B, Hq, D = inp["q"].shape
    Hkv, T_cap = cache["k_codes"].shape[1], cache["k_codes"].shape[2]
    out = torch.empty(B, Hq, D, dtype=torch.float32, device="cuda")
    mask = torch.zeros(B, Hq, T_cap, dtype=torch.uint8, device="cuda") if want_mask else None
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    nb = lkv.lkv_decode_workspace_bytes((kb, vb, G), B, Hq, Hkv, T_cap, D)
    if ws is None:
        ws = buffers.alloc_workspace(nb)
    lkv.lkv_decode_attention((kb, vb, G), B, Hq, Hkv, T_cap, D, dev(inp["seq_lens"]), dev(inp["q"]),
                             cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"],
                             softmax_scale, tau, out, mask, counts, ws, ws.numel())
    torch.cuda.synchronize()
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_OK
    return out.cpu().numpy(), (mask.cpu().numpy() if want_mask else None), counts.cpu().numpy()


def oracle_inputs(inp):
    return (W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"]), W.bf16_bits(inp["q"]),
            inp["seq_lens"].numpy())


def vmax(inp):
    v = inp["v"].float()
    return float(v.abs().max()) if v.numel() else 1.0


def assert_attention_close(got, want, v_max, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), what
    err = got - want
    nrm = np.linalg.norm(want)
    rel = np.linalg.norm(err) / nrm if nrm > 0 else np.linalg.norm(err)
    mx = np.max(np.abs(err)) if err.size else 0.0
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_PER_VMAX * v_max, f"{what}: max-abs {mx:.3e} > {MAX_ABS_PER_VMAX} * {v_max}"
    return rel, mx


def assert_masks_match(got, want, p, tau, seq_lens, what=""):
    """Skip masks equal outside |p - tau| < 1e-7, over valid positions only."""
    B, Hq, T_cap = want.shape
    valid = np.arange(T_cap)[None, None, :] < np.asarray(seq_lens)[:, None, None]
    band = np.abs(p - tau) < TIE_BAND
    bad = (got != want) & valid & ~band
    assert not bad.any(), f"{what}: {int(bad.sum())} skip decisions differ outside the tie band"
    return int(((got != want) & valid).sum())
