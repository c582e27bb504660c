"""lkv_decode_attention on the GPU vs the CPU oracle: attention outputs within
rel-L2 1e-5 and max-abs 5e-5 * max|V|, skip masks equal outside the 1e-7 tie
band around tau, skip counts consistent ("Super KV Compression" §第三层)."""
import numpy as np
import pytest
import torch

from gpu_helpers import (assert_attention_close, assert_masks_match, dev, gpu_decode, gpu_quantize,
                         oracle_inputs, vmax)
from quantized_kv_cache_lkv_b200 import buffers, lkv
from quantized_kv_cache_lkv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def run_case(orc, cfg, kb, vb, tau, seq_lens=None, batches=None, inp=None):
    """Quantize + decode the whole batch on the GPU; check the batches listed
    (all by default) against the oracle, which quantizes from bf16 itself."""
    if inp is None:
        inp = W.make_inputs(cfg, seq_lens=seq_lens)
    cache = gpu_quantize(kb, vb, cfg.G, inp)
    out, mask, counts = gpu_decode(kb, vb, cfg.G, inp, cache, cfg.softmax_scale, tau)
    bsel = list(range(cfg.B)) if batches is None else list(batches)
    sub = {key: inp[key][bsel].contiguous() for key in ("q", "k", "v", "seq_lens")}
    k, v, q, sl = oracle_inputs(sub)
    ocache = orc.quantize_kv(kb, vb, cfg.G, k, v, sl)
    o_out, o_mask, o_counts, p = orc.decode_attention(kb, vb, cfg.G, sl, q, ocache, cfg.softmax_scale, tau,
                                                      want_p=True)
    what = f"{cfg.name} K{kb}V{vb} tau={tau}"
    assert_attention_close(out[bsel], o_out, vmax(sub), what)
    n_band = assert_masks_match(mask[bsel], o_mask, p, np.float32(tau), sl, what)
    valid = np.arange(mask.shape[2])[None, None, :] < inp["seq_lens"].numpy()[:, None, None]
    assert counts[0] == int((mask * valid).sum())        # counts agree with the mask written
    if batches is None:
        assert abs(int(counts[0]) - int(o_counts[0])) <= n_band
        if n_band == 0:
            assert counts.tolist() == o_counts.tolist()
    return out, mask, counts


def test_decode_config1_tiny(orc):
    run_case(orc, W.CONFIGS[1], 6, 4, 0.0)


@pytest.mark.parametrize("r", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_gqa_ratios_ragged(orc, r, D):
    """Several chunks plus a ragged tail, lengths 0 and 1, every GQA ratio."""
    G = 32 if D == 64 else 64
    cfg = W.Config("ragged", B=4, Hq=2 * r, Hkv=2, D=D, T_cap=600, G=G, bits=[(6, 4)], hh_frac=0.01,
                   seed=10 * r + D)
    sl = torch.tensor([600, 1, 0, 333], dtype=torch.int32)
    for tau in (0.0, 1e-3):
        out, _, _ = run_case(orc, cfg, 6, 4, tau, seq_lens=sl)
        assert np.all(out[2] == 0.0)


@pytest.mark.parametrize("kb,vb", [(8, 8), (6, 4), (4, 4), (4, 2), (2, 2), (2, 8), (8, 6),
                                   (16, 16), (16, 4), (6, 16), (16, 8)])
def test_decode_bit_widths(orc, kb, vb):
    cfg = W.scaled(W.CONFIGS[4], B=3, T_cap=520, seq_lo=100, seq_hi=520, seed=40 + kb + vb)
    run_case(orc, cfg, kb, vb, 0.0)
    run_case(orc, cfg, kb, vb, 2e-3)


@pytest.mark.parametrize("r", [1, 2, 4, 8])
@pytest.mark.parametrize("kb,vb", [(16, 16), (16, 4), (6, 16)])
def test_decode_passthrough_width_gqa(orc, r, kb, vb):
    """The 16-bit width through every GQA ratio (groups of 8 take the
    three-launch path), D 64 and 128, ragged lengths with 0 and 1."""
    for D, G in ((128, 64), (64, 32)):
        cfg = W.Config("pass", B=4, Hq=2 * r, Hkv=2, D=D, T_cap=600, G=G, bits=[(kb, vb)], hh_frac=0.01,
                       seed=7 * r + kb + vb + D)
        sl = torch.tensor([600, 1, 0, 333], dtype=torch.int32)
        for tau in (0.0, 1e-3):
            out, _, _ = run_case(orc, cfg, kb, vb, tau, seq_lens=sl)
            assert np.all(out[2] == 0.0)


def test_per_layer_bit_policy_two_layers(orc):
    """A per-layer width policy is a table on the caller's side: an outlier
    layer kept at 16 bits (K16V16) and an ordinary layer at K6V4, each with
    its own cache, decoded one after the other with one workspace sized for
    the larger of the two; each layer matches the oracle at its own width
    ("Super KV Compression" §第一层: outlier layers stay in 16-bit floating
    point, the others take K6V4)."""
    policy = {0: (16, 16), 1: (6, 4)}
    base = W.scaled(W.CONFIGS[2], B=2, T_cap=1024)
    layers = {layer: W.make_inputs(W.scaled(base, seed=200 + layer)) for layer in policy}
    B, Hq, Hkv, D, T, G = base.B, base.Hq, base.Hkv, base.D, base.T_cap, base.G
    nb = max(lkv.lkv_decode_workspace_bytes((kb, vb, G), B, Hq, Hkv, T, D) for kb, vb in policy.values())
    ws = buffers.alloc_workspace(nb)
    caches = {layer: gpu_quantize(kb, vb, G, layers[layer]) for layer, (kb, vb) in policy.items()}
    for step in range(2):
        for layer, (kb, vb) in policy.items():
            inp = layers[layer]
            got, _, counts = gpu_decode(kb, vb, G, inp, caches[layer], base.softmax_scale, base.tau,
                                        want_mask=False, ws=ws)
            k, v, q, sl = oracle_inputs(inp)
            want, _, o_counts = orc.decode_attention(kb, vb, G, sl, q, orc.quantize_kv(kb, vb, G, k, v, sl),
                                                     base.softmax_scale, base.tau, want_mask=False)
            assert_attention_close(got, want, vmax(inp), f"layer {layer} K{kb}V{vb} step {step}")
    # the outlier layer's cache is the bf16 cache itself; the other is 3.2x smaller in codes
    c0, c1 = caches[0], caches[1]
    assert c0["k_codes"].shape[-1] == 2 * D and c1["k_codes"].shape[-1] + c1["v_codes"].shape[-1] == 10 * D // 8


@pytest.mark.parametrize("tau", [1e-4, 1e-2, 0.5])
def test_decode_skip_thresholds(orc, tau):
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=1024, seed=77)
    run_case(orc, cfg, 6, 4, tau)


def test_decode_tau_above_every_probability_gives_zero(orc):
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=300, seed=5)
    out, mask, counts = run_case(orc, cfg, 6, 4, 1.5)
    assert np.all(out == 0.0) and counts.tolist() == [2 * 32 * 300, 2 * 8 * 300]


def test_decode_more_units_than_threads(orc):
    """576 (sequence, KV head) units, more than one CTA's threads: the unit
    list takes its two-pass path; ragged lengths including 0, every
    sequence against the oracle."""
    cfg = W.scaled(W.CONFIGS[2], B=72, T_cap=320, seq_lo=0, seq_hi=320, seq="uniform", seed=91)
    out, _, _ = run_case(orc, cfg, 6, 4, 1e-3)
    zero = np.nonzero(W.make_inputs(cfg)["seq_lens"].numpy() == 0)[0]
    assert np.all(out[zero] == 0.0)


def test_decode_kept_list_overflow_falls_back(orc):
    """One CTA per unit (112 units) with 4096 rows each and tau 1e-9: nearly
    every row is kept, more than the 2048 one CTA can list, so the sparse
    pass falls back to the per-piece scan; outputs, masks and counts still
    match the oracle."""
    cfg = W.scaled(W.CONFIGS[2], B=14, T_cap=4096, seed=93)
    out, mask, counts = run_case(orc, cfg, 6, 4, 1e-9)
    assert counts[1] < 14 * 8 * 4096 // 10     # most rows kept by some head


def test_decode_capacity_invariance(orc):
    """The same tokens in a larger cache (more chunks launched, most of them
    empty) give the same skip set and outputs within tolerance."""
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=700, seed=12)
    inp = W.make_inputs(cfg)
    big = dict(inp)
    for key in ("k", "v"):
        t = torch.zeros(2, 8, 1300, 128, dtype=torch.bfloat16)
        t[:, :, :700] = inp[key]
        big[key] = t
    o1, m1, c1 = run_case(orc, cfg, 6, 4, 1e-4, inp=inp)
    cfg2 = W.scaled(cfg, T_cap=1300)
    o2, m2, c2 = run_case(orc, cfg2, 6, 4, 1e-4, inp=big)
    np.testing.assert_array_equal(m1, m2[:, :, :700])
    assert c1.tolist() == c2.tolist()
    assert_attention_close(o2, o1, vmax(inp), "invariance")


def test_decode_workspace_reuse_is_deterministic(orc):
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=900, seed=8)
    inp = W.make_inputs(cfg)
    cache = gpu_quantize(6, 4, cfg.G, inp)
    ws = buffers.alloc_workspace(lkv.lkv_decode_workspace_bytes((6, 4, 64), 2, 32, 8, 900, 128))
    a = gpu_decode(6, 4, 64, inp, cache, cfg.softmax_scale, 1e-4, ws=ws)
    b = gpu_decode(6, 4, 64, inp, cache, cfg.softmax_scale, 1e-4, ws=ws)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_decode_bad_length_sets_device_status(orc):
    cfg = W.Config("bad", B=2, Hq=4, Hkv=2, D=64, T_cap=64, G=32, bits=[(6, 4)], seed=1)
    inp = W.make_inputs(cfg)
    cache = gpu_quantize(6, 4, 32, inp)
    inp["seq_lens"] = torch.tensor([64, 65], dtype=torch.int32)
    nb = lkv.lkv_decode_workspace_bytes((6, 4, 32), 2, 4, 2, 64, 64)
    ws = buffers.alloc_workspace(nb)
    out = torch.empty(2, 4, 64, device="cuda")
    lkv.lkv_decode_attention((6, 4, 32), 2, 4, 2, 64, 64, dev(inp["seq_lens"]), dev(inp["q"]),
                             cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"],
                             cfg.softmax_scale, 0.0, out, None, None, ws, ws.numel())
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_ERR_INVALID_ARG
    assert torch.isfinite(out).all()          # clamped to T_cap, no fault
    lkv.lkv_workspace_reset(ws, ws.numel())
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_OK


def test_decode_bounded_wait_times_out(orc):
    """A unit split over several CTAs waits for its neighbours' statistics.
    Plant a missing arrival on the host (the unit's arrival counter starts
    far below its target) with a 1 ms limit: the call must end with
    LKV_ERR_TIMEOUT and finite outputs, and after a reset the same workspace
    gives correct results."""
    cfg = W.Config("wait", B=1, Hq=4, Hkv=1, D=128, T_cap=8192, G=64, bits=[(6, 4)], seed=6)
    inp = W.make_inputs(cfg)
    cache = gpu_quantize(6, 4, 64, inp)
    nb = lkv.lkv_decode_workspace_bytes((6, 4, 64), 1, 4, 1, 8192, 128)
    ws = buffers.alloc_workspace(nb)
    ws[8:16].view(torch.int64).fill_(1_000_000)          # wait limit: 1 ms
    ws[256:260].view(torch.int32).fill_(-(1 << 30))      # arrival counter of unit 0 (first after the header)
    out = torch.empty(1, 4, 128, device="cuda")
    lkv.lkv_decode_attention((6, 4, 64), 1, 4, 1, 8192, 128, dev(inp["seq_lens"]), dev(inp["q"]),
                             cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"],
                             cfg.softmax_scale, 1e-4, out, None, None, ws, ws.numel())
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_ERR_TIMEOUT
    assert torch.isfinite(out).all()
    lkv.lkv_workspace_reset(ws, ws.numel())
    got, _, _ = gpu_decode(6, 4, 64, inp, cache, cfg.softmax_scale, 1e-4, ws=ws)
    k, v, q, sl = oracle_inputs(inp)
    want, _, _ = orc.decode_attention(6, 4, 64, sl, q, orc.quantize_kv(6, 4, 64, k, v, sl),
                                      cfg.softmax_scale, 1e-4)
    assert_attention_close(got, want, vmax(inp), "after reset")


@pytest.mark.slow
def test_decode_llama8b_full_size_sampled(orc):
    """The Llama-3.1-8B-shaped workload at full size (B16, 32q/8kv, D128,
    T8192, 1% heavy hitters, tau 1e-4) in the bench's launch, every sequence
    against the oracle: outputs, skip masks, and both skip counts exactly
    when no probability falls in the tie band."""
    out, mask, counts = run_case(orc, W.CONFIGS[2], 6, 4, 1e-4)
    assert 0 < counts[1] < 16 * 8 * 8192


@pytest.mark.slow
def test_decode_long_context_full_size(orc):
    run_case(orc, W.CONFIGS[3], 6, 4, 1e-5)


@pytest.mark.slow
def test_decode_long_context_groups_of_eight(orc):
    """The long-context decode (B1, T131072, tau 1e-5, 0.1% heavy hitters)
    with 64 query heads over 8 KV heads: groups of 8 query heads per KV head
    take the three-launch path; every head against the oracle."""
    cfg = W.scaled(W.CONFIGS[3], name="long_r8", Hq=64, seed=12)
    run_case(orc, cfg, 6, 4, 1e-5)


@pytest.mark.slow
@pytest.mark.parametrize("kb,vb", [(8, 8), (6, 4), (4, 4), (4, 2)])
def test_decode_sweep_full_size_sampled(orc, kb, vb):
    cfg = W.CONFIGS[4]
    run_case(orc, cfg, kb, vb, 0.0)


@pytest.mark.parametrize("r", [1, 2, 4, 8])
def test_decode_attention_mass(orc, r):
    """lkv_decode_attention_mass: the group's mean softmax probability per
    token ("Super KV Compression" §第二层 ranks tokens by it) matches the
    oracle's within 1e-4 relative (an fp32 logit carries an absolute error of
    order 1e-5 in base 2, which moves exp2 by about 7e-6 relative per unit
    of error, plus the error of the shared sum); every other output is
    bit-identical to
    lkv_decode_attention; slots beyond T_b are left untouched."""
    cfg = W.Config("mass", B=3, Hq=2 * r, Hkv=2, D=128, T_cap=700, G=64, bits=[(6, 4)], hh_frac=0.01,
                   seed=50 + r)
    sl = torch.tensor([700, 1, 333], dtype=torch.int32)
    inp = W.make_inputs(cfg, seq_lens=sl)
    cache = gpu_quantize(6, 4, 64, inp)
    tau = 1e-3
    want_out, want_mask, want_counts = gpu_decode(6, 4, 64, inp, cache, cfg.softmax_scale, tau)
    out = torch.empty(3, 2 * r, 128, device="cuda")
    mask = torch.zeros(3, 2 * r, 700, dtype=torch.uint8, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    mass = torch.full((3, 2, 700), -1.0, device="cuda")
    nb = lkv.lkv_decode_workspace_bytes((6, 4, 64), 3, 2 * r, 2, 700, 128)
    ws = buffers.alloc_workspace(nb)
    lkv.lkv_decode_attention_mass((6, 4, 64), 3, 2 * r, 2, 700, 128, dev(inp["seq_lens"]), dev(inp["q"]),
                                  cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"],
                                  cfg.softmax_scale, tau, out, mask, counts, mass, ws, nb)
    torch.cuda.synchronize()
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_OK
    np.testing.assert_array_equal(out.cpu().numpy(), want_out)
    np.testing.assert_array_equal(mask.cpu().numpy(), want_mask)
    assert counts.cpu().tolist() == want_counts.tolist()
    k, v, q, s = oracle_inputs(inp)
    ocache = orc.quantize_kv(6, 4, 64, k, v, s)
    _, _, _, p = orc.decode_attention(6, 4, 64, s, q, ocache, cfg.softmax_scale, tau, want_p=True)
    want = orc.attention_mass(p, 2, s)
    got = mass.cpu().numpy()
    for b in range(3):
        T = int(s[b])
        np.testing.assert_allclose(got[b, :, :T], want[b, :, :T], rtol=1e-4, atol=1e-12)
        assert np.all(got[b, :, T:] == -1.0)


def test_decode_mass_feeds_the_tiers(orc):
    """One step of the attention-tiered cache driven by its own decode: the
    mass from lkv_decode_attention_mass classified on the GPU gives the
    oracle's tiers, except for masses within 1e-4 relative of a threshold."""
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=1024, seed=61)
    inp = W.make_inputs(cfg)
    cache = gpu_quantize(6, 4, 64, inp)
    nb = lkv.lkv_decode_workspace_bytes((6, 4, 64), 2, 32, 8, 1024, 128)
    ws = buffers.alloc_workspace(nb)
    out = torch.empty(2, 32, 128, device="cuda")
    mass = torch.zeros(2, 8, 1024, device="cuda")
    sl = dev(inp["seq_lens"])
    lkv.lkv_decode_attention_mass((6, 4, 64), 2, 32, 8, 1024, 128, sl, dev(inp["q"]), cache["k_codes"],
                                  cache["k_sz"], cache["v_codes"], cache["v_sz"], cfg.softmax_scale, 1e-4, out,
                                  None, None, mass, ws, nb)
    t = buffers.alloc_tiers(2, 8, 1024, "cuda", zero=True)
    lo, hi = 1e-4, 1e-2
    lkv.lkv_tier_classify(2, 8, 1024, sl, mass, lo, hi, t["tier"], t["counts"], t["pos_a"], t["pos_b"])
    torch.cuda.synchronize()
    k, v, q, s = oracle_inputs(inp)
    ocache = orc.quantize_kv(6, 4, 64, k, v, s)
    _, _, _, p = orc.decode_attention(6, 4, 64, s, q, ocache, cfg.softmax_scale, 1e-4, want_p=True)
    m_or = orc.attention_mass(p, 8, s)
    tier_or, _, _, _ = orc.tier_classify(s, m_or.astype(np.float32), lo, hi)
    near = (np.abs(m_or - lo) <= 1e-4 * lo) | (np.abs(m_or - hi) <= 1e-4 * hi)
    got = t["tier"].cpu().numpy()
    assert np.all((got == tier_or) | near)
    assert (got == 2).sum() > 0 and (got == 1).sum() > 0 and (got == 0).sum() > 0
