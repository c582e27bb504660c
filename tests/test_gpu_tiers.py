"""Attention-tiered cache on the GPU vs the CPU oracle ("Super KV
Compression" §第二层): tiers, counts and positions bit-exact, repacked
segments bit-exact, tiered attention within the attention tolerance."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_attention_close, dev, gpu_decode, gpu_quantize, oracle_inputs, vmax
from quantized_kv_cache_lkv_b200 import buffers, lkv
from quantized_kv_cache_lkv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def gpu_classify(inp, tau_low, tau_high):
    B, Hkv, T_cap = inp["mass"].shape
    t = buffers.alloc_tiers(B, Hkv, T_cap, zero=True)
    lkv.lkv_tier_classify(B, Hkv, T_cap, dev(inp["seq_lens"]), dev(inp["mass"]), tau_low, tau_high,
                          t["tier"], t["counts"], t["pos_a"], t["pos_b"])
    torch.cuda.synchronize()
    return t


def gpu_repack(inp, G, t):
    B, Hkv, T_cap, D = inp["k"].shape
    A, Bs = buffers.alloc_segments(G, B, Hkv, T_cap, D, zero=True)
    lkv.lkv_tier_repack(B, Hkv, T_cap, D, G, dev(inp["k"]), dev(inp["v"]), t["counts"], t["pos_a"],
                        t["pos_b"], A, Bs)
    torch.cuda.synchronize()
    return A, Bs


def gpu_tiered_attention(inp, G, t, A, Bs, scale, tau):
    B, Hq, D = inp["q"].shape
    Hkv, T_cap = inp["k"].shape[1], inp["k"].shape[2]
    out = torch.empty(B, Hq, D, device="cuda")
    cnt = torch.zeros(2, dtype=torch.int64, device="cuda")
    ws = buffers.alloc_workspace(lkv.lkv_tiered_workspace_bytes(B, Hq, Hkv, T_cap, D, G))
    lkv.lkv_tiered_attention(B, Hq, Hkv, T_cap, D, G, t["counts"], dev(inp["q"]), A, Bs, scale, tau, out,
                             cnt, ws, ws.numel())
    torch.cuda.synchronize()
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_OK
    return out.cpu().numpy(), cnt.cpu().numpy()


def check_tiers(t, want, seq_lens):
    tier, counts, p2, p1 = want
    np.testing.assert_array_equal(t["tier"].cpu().numpy(), tier)
    c = t["counts"].cpu().numpy()
    np.testing.assert_array_equal(c, counts)
    ga, gb = t["pos_a"].cpu().numpy(), t["pos_b"].cpu().numpy()
    B, Hkv, _ = tier.shape
    for b in range(B):
        for g in range(Hkv):
            n2, n1 = counts[b, g]
            np.testing.assert_array_equal(ga[b, g, :n2], p2[b, g, :n2])
            np.testing.assert_array_equal(gb[b, g, :n1], p1[b, g, :n1])


def check_segments(A, Bs, oA, oB, counts):
    for seg, want, ci in ((A, oA, 0), (Bs, oB, 1)):
        for key in ("k_codes", "k_sz", "v_codes", "v_sz"):
            g = seg[key].cpu().numpy()
            w = want[key]
            B, Hkv = counts.shape[:2]
            for b in range(B):
                for h in range(Hkv):
                    n = counts[b, h, ci]
                    gb, wb = g[b, h, :n], w[b, h, :n]
                    if key.endswith("sz"):
                        gb, wb = gb.view(np.uint32), wb.view(np.uint32)
                    assert np.array_equal(gb, wb), (key, b, h, ci)


def tiered_case(orc, cfg, tau_low, tau_high, tau=0.0, batches=None):
    inp = W.make_inputs(cfg, with_mass=True)
    t = gpu_classify(inp, tau_low, tau_high)
    A, Bs = gpu_repack(inp, cfg.G, t)
    out, cnt = gpu_tiered_attention(inp, cfg.G, t, A, Bs, cfg.softmax_scale, tau)
    bsel = list(range(cfg.B)) if batches is None else list(batches)
    sub = {key: inp[key][bsel].contiguous() for key in ("q", "k", "v", "seq_lens", "mass")}
    k, v, q, sl = oracle_inputs(sub)
    want = orc.tier_classify(sl, sub["mass"].numpy(), tau_low, tau_high)
    tsub = {key: val[bsel] for key, val in t.items()}
    check_tiers(tsub, want, sl)
    oA, oB = orc.tier_repack(cfg.G, k, v, want[1], want[2], want[3])
    Asub = {key: val[bsel] for key, val in A.items()}
    Bsub = {key: val[bsel] for key, val in Bs.items()}
    check_segments(Asub, Bsub, oA, oB, want[1])
    o_out, o_cnt = orc.tiered_attention(cfg.G, want[1], q, oA, oB, cfg.softmax_scale, tau)
    assert_attention_close(out[bsel], o_out, vmax(sub), f"tiered {cfg.name}")
    if batches is None and tau == 0.0:
        assert cnt.tolist() == [0, 0] == o_cnt.tolist()
    return inp, t, A, Bs, out


def test_tier_boundaries_exact(orc):
    lo, hi = np.float32(1e-4), np.float32(1e-2)
    vals = np.array([hi, np.nextafter(hi, np.float32(1)), lo, np.nextafter(lo, np.float32(0)), 0.5, 0.0,
                     np.nan, 3e-3], np.float32)
    T_cap = 16
    mass = torch.full((1, 2, T_cap), 0.9)
    mass[0, :, :8] = torch.from_numpy(vals)
    inp = {"mass": mass, "seq_lens": torch.tensor([8], dtype=torch.int32)}
    t = gpu_classify(inp, lo, hi)
    check_tiers(t, orc.tier_classify(np.array([8], np.int32), mass.numpy(), lo, hi), [8])
    assert t["tier"][0, 0, :8].tolist() == [1, 2, 1, 0, 2, 0, 0, 1]


def test_tiered_small_ragged(orc):
    cfg = W.scaled(W.CONFIGS[5], B=3, T_cap=9000, seq_lo=300, seq_hi=9000, seed=31)
    tiered_case(orc, cfg, 1e-4, 1e-2)
    tiered_case(orc, cfg, 1e-4, 1e-2, tau=1e-3)


def test_tiered_d64_r2(orc):
    cfg = W.Config("t64", B=2, Hq=4, Hkv=2, D=64, T_cap=2048, G=32, bits=[(6, 4)], seq="uniform",
                   seq_lo=1, seq_hi=2048, seed=9)
    tiered_case(orc, cfg, 2e-4, 5e-3)


def test_tiered_everything_kept_equals_plain_k6v4(orc):
    """tau_low = 0 and tau_high = inf keep every token at V4: the tiered path
    then equals plain K6V4 decode."""
    cfg = W.scaled(W.CONFIGS[5], B=2, T_cap=1500, seq_lo=700, seq_hi=1500, seed=19)
    inp, t, A, Bs, out = tiered_case(orc, cfg, 0.0, float("inf"))
    cache = gpu_quantize(6, 4, cfg.G, inp)
    plain, _, _ = gpu_decode(6, 4, cfg.G, inp, cache, cfg.softmax_scale, 0.0)
    assert_attention_close(out, plain, vmax(inp), "tiered vs plain")


def test_tiered_all_evicted_gives_zero(orc):
    cfg = W.scaled(W.CONFIGS[5], B=2, T_cap=1024, seq_lo=1024, seq_hi=1024, seed=2)
    inp, t, _, _, out = tiered_case(orc, cfg, 2.0, 3.0)
    assert int(t["counts"].sum()) == 0 and np.all(out == 0.0)


def test_tiered_decode_composite_equals_stages(orc):
    cfg = W.scaled(W.CONFIGS[5], B=2, T_cap=4096, seq_lo=1024, seq_hi=4096, seed=23)
    inp, t, A, Bs, out = tiered_case(orc, cfg, cfg.tau_low, cfg.tau_high)
    B, Hq, D = inp["q"].shape
    Hkv, T_cap = inp["k"].shape[1], inp["k"].shape[2]
    t2 = buffers.alloc_tiers(B, Hkv, T_cap, zero=True)
    A2, B2 = buffers.alloc_segments(cfg.G, B, Hkv, T_cap, D, zero=True)
    out2 = torch.empty(B, Hq, D, device="cuda")
    ws = buffers.alloc_workspace(lkv.lkv_tiered_workspace_bytes(B, Hq, Hkv, T_cap, D, cfg.G))
    lkv.lkv_tiered_decode(B, Hq, Hkv, T_cap, D, cfg.G, dev(inp["seq_lens"]), dev(inp["mass"]), cfg.tau_low,
                          cfg.tau_high, dev(inp["k"]), dev(inp["v"]), dev(inp["q"]), t2["tier"], t2["counts"],
                          t2["pos_a"], t2["pos_b"], A2, B2, cfg.softmax_scale, 0.0, out2, None, ws, ws.numel())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out2.cpu().numpy(), out)
    assert torch.equal(t2["tier"], t["tier"]) and torch.equal(t2["counts"], t["counts"])


@pytest.mark.slow
def test_tiered_full_size_sampled(orc):
    """The tiered workload at full size (B32, context log-uniform in
    [1024, 32768], Zipf(1.1) mass); sequences 0, 17 and 31 checked."""
    tiered_case(orc, W.CONFIGS[5], W.CONFIGS[5].tau_low, W.CONFIGS[5].tau_high, batches=[0, 17, 31])


@pytest.mark.parametrize("B", [512, 1040])
def test_repack_both_row_layouts(orc, B):
    """Up to 8192 (segment, unit) pairs the repack deals all kept rows evenly
    over resident blocks; past that it gives each pair its own blocks.  B512
    (8192 pairs) and B1040 (16640 pairs) with 8 KV heads and short ragged
    contexts take one layout each; segments are bit-exact with the oracle
    on sampled sequences."""
    cfg = W.scaled(W.CONFIGS[5], B=B, T_cap=24, seq_lo=1, seq_hi=24, seed=71 + B)
    tiered_case(orc, cfg, 2e-3, 5e-2, batches=[0, B // 2 + 1, B - 1])
