"""Pins for the CPU oracle: each test checks it against something other than
itself -- a closed form, brute force, a float64 library softmax, or a value
the pages print.  No GPU needed.

Sources: "Super KV Compression: 突破LLM推理内存瓶颈的三层压缩架构解析"
(§第一层 K6V4 asymmetric quantization, §第二层 attention tiers, §第三层
sparse-V skip, comparison table) and "TurboQuant：将LLM KV缓存压缩5-7倍的
突破性技术" (§TurboQuant的核心创新: asymmetric, group-wise quantization).
"""
import math
import os

import numpy as np
import pytest
import torch

from quantized_kv_cache_lkv_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = (2, 4, 6, 8)


def f32(x):
    return np.float32(x)


def ulp(x):
    x = np.float32(abs(x))
    return np.float32(np.spacing(x)) if x != 0 else np.float32(np.finfo(np.float32).tiny)


def bf16_round(a):
    """fp32 -> bf16 -> fp32 (RNE), via torch."""
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def random_groups(rng, n, G):
    """Groups with varied ranges: normal, scaled, outliers, tiny spread, large
    magnitude, spreads so small that qmax / d overflows fp32 (subnormal and
    near-subnormal values), and spans of +-1e38..3e38 whose d overflows."""
    out = []
    for i in range(n):
        kind = i % 7
        x = rng.standard_normal(G).astype(np.float32)
        if kind == 1:
            x *= np.float32(rng.uniform(0.01, 100))
        elif kind == 2:
            x[rng.integers(G)] *= 15
        elif kind == 3:
            x = np.float32(rng.uniform(-50, 50)) + x * np.float32(0.3)
        elif kind == 4:
            x = x * np.float32(1e20)
        elif kind == 5:
            if i % 2:  # subnormal values
                x = x * np.float32(10.0 ** rng.uniform(-40, -37.5))
            else:  # a few steps around a near-subnormal base
                x = np.float32(2.0 ** -120) + rng.integers(-2, 3, G).astype(np.float32) * np.float32(2.0 ** -127)
        elif kind == 6:
            x = rng.uniform(-3.0, 3.0, G).astype(np.float32) * np.float32(1e38)
            x[0] = np.float32(rng.uniform(1.0, 3.0) * 1e38)
            x[1] = -np.float32(rng.uniform(1.0, 3.0) * 1e38)
        out.append(bf16_round(x))
    return out


def p1_bound(x, s, bits):
    """P1: scale/2, plus the storage precision of the scale (a subnormal scale
    keeps few bits: code * scale may miss code * d/qmax by (qmax/2) ulp(scale)),
    plus the fp32 rounding of the formula, 2 ulp(max(|mn|, |mx|))."""
    qmax = (1 << bits) - 1
    mag = max(abs(float(x.min())), abs(float(x.max())))
    return float(s) / 2 + (qmax / 2 + 1) * float(ulp(s)) + 2 * float(ulp(mag))


# ---------------------------------------------------------------- bit layout

def test_pack_golden_fixture(orc):
    """Rows worked by hand (tests/golden/pack_lsb_first.txt)."""
    n = 0
    for line in open(os.path.join(GOLDEN, "pack_lsb_first.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        b, codes, hexes = [s.strip() for s in line.split("|")]
        b = int(b)
        codes = np.array([int(c) for c in codes.split()], np.uint32)
        want = np.array([int(h, 16) for h in hexes.split()], np.uint8)
        got = orc.pack_row(codes, b)
        assert got.tolist() == want.tolist(), (b, codes)
        assert orc.unpack_row(want, codes.size, b).tolist() == codes.tolist()
        n += 1
    assert n >= 6


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("D", [64, 128])
def test_pack_roundtrip_bruteforce(orc, bits, D):
    """Every code value round-trips, and the bytes read as one little-endian
    integer give code j at bit offset j*bits (Python big-int arithmetic)."""
    rng = np.random.default_rng(bits * 1000 + D)
    qmax = (1 << bits) - 1
    for trial in range(4):
        codes = rng.integers(0, qmax + 1, D).astype(np.uint32)
        codes[: min(D, qmax + 1)] = np.arange(min(D, qmax + 1))  # all values appear
        rng.shuffle(codes)
        row = orc.pack_row(codes, bits)
        assert row.size == D * bits // 8
        big = int.from_bytes(row.tobytes(), "little")
        assert [(big >> (j * bits)) & qmax for j in range(D)] == codes.tolist()
        assert orc.unpack_row(row, D, bits).tolist() == codes.tolist()


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("bits", BITS)
def test_quantize_error_bound(orc, bits):
    """P1: |x - xhat| <= scale/2 + (qmax/2 + 1) ulp(scale) + 2 ulp(max(|mn|,
    |mx|)) for every element, and every reconstruction finite (the
    quantization error bound the tier thresholds are derived from, Super KV
    Compression §第二层), for every kind of finite group."""
    rng = np.random.default_rng(bits)
    for x in random_groups(rng, 200, 64):
        codes, s, z = orc.quantize_group(x, bits)
        assert codes.max() <= (1 << bits) - 1
        xh = np.array([orc.dequant(c, s, z) for c in codes], np.float32)
        assert np.all(np.isfinite(xh)) and np.isfinite(s)
        bound = p1_bound(x, s, bits)
        assert np.all(np.abs(x.astype(np.float64) - xh.astype(np.float64)) <= bound), (bits, s)


@pytest.mark.parametrize("bits", BITS)
def test_quantize_is_nearest_level(orc, bits):
    """Brute force over all 2^bits levels: the chosen code's reconstruction is
    the nearest level to within the fp32 rounding of the formula."""
    rng = np.random.default_rng(100 + bits)
    qmax = (1 << bits) - 1
    for x in random_groups(rng, 60, 32):
        codes, s, z = orc.quantize_group(x, bits)
        levels = np.array([orc.dequant(c, s, z) for c in range(qmax + 1)], np.float64)
        mag = max(abs(float(x.min())), abs(float(x.max())))
        slack = 4 * float(ulp(mag)) + 1e-7 * float(s) + qmax * float(ulp(s))
        for xi, c in zip(x.astype(np.float64), codes):
            best = np.min(np.abs(levels - xi))
            assert abs(levels[c] - xi) <= best + slack


@pytest.mark.parametrize("bits", BITS)
def test_group_min_and_max(orc, bits):
    """P2: the group minimum reconstructs bit-exactly (code 0 -> zero = mn);
    the maximum gets code qmax and reconstructs exactly up to the fp32
    rounding of scale = d/qmax and of the final fused multiply-add: within
    (qmax/2) ulp(scale) + 4 ulp(max(|mn|, |mx|)), since d <= 2 max(|mn|, |mx|)."""
    rng = np.random.default_rng(200 + bits)
    qmax = (1 << bits) - 1
    for x in random_groups(rng, 100, 64):
        codes, s, z = orc.quantize_group(x, bits)
        i_mn, i_mx = int(np.argmin(x)), int(np.argmax(x))
        assert codes[i_mn] == 0
        assert orc.dequant(codes[i_mn], s, z) == x[i_mn] + np.float32(0.0)
        assert z == x[i_mn]
        if x.max() == x.min():
            continue  # a constant group has no separate maximum
        assert codes[i_mx] == qmax
        mag = max(abs(float(x.min())), abs(float(x.max())))
        xm = float(orc.dequant(codes[i_mx], s, z))
        assert abs(xm - float(x[i_mx])) <= qmax / 2 * float(ulp(s)) + 4 * float(ulp(mag))


@pytest.mark.parametrize("bits", BITS)
def test_constant_group(orc, bits):
    """d == 0: scale 0, every code 0, reconstruction = the constant exactly."""
    for c in (0.0, -0.0, 1.5, -3.25e5, 7e-30):
        x = np.full(32, c, np.float32)
        codes, s, z = orc.quantize_group(x, bits)
        assert s == 0.0 and np.all(codes == 0)
        assert np.float32(z) == np.float32(c)
        assert np.signbit(z) == (c < 0)  # a minus zero is stored as plus zero
        assert orc.dequant(0, s, z) == np.float32(c)


@pytest.mark.parametrize("bits", BITS)
def test_arithmetic_progression_exact(orc, bits):
    """Values mn + k*s with s = d/qmax exactly representable get code k."""
    qmax = (1 << bits) - 1
    rng = np.random.default_rng(300 + bits)
    for step, base in ((0.5, -3.0), (0.25, 10.0), (1.0, 0.0), (2.0 ** -6, -1.0)):
        k = rng.integers(0, qmax + 1, 64)
        k[0], k[1] = 0, qmax
        x = (np.float32(base) + k.astype(np.float32) * np.float32(step)).astype(np.float32)
        codes, s, z = orc.quantize_group(x, bits)
        assert s == np.float32(step) and z == np.float32(base)
        assert codes.tolist() == k.tolist()


@pytest.mark.parametrize("bits", BITS)
def test_tiny_range_progression_exact(orc, bits):
    """A spread so small that qmax / d overflows fp32: x_k = mn + k * 2^-140
    (fp32 subnormal steps), d = qmax * 2^-140.  The rescaled formula gives
    code k exactly, scale = 2^-140 exactly, and every x_k reconstructs."""
    qmax = (1 << bits) - 1
    step = np.float32(2.0 ** -140)
    for base in (0.0, -(2.0 ** -135), 2.0 ** -130):
        k = np.arange(qmax + 1)[::-1].copy()
        x = (np.float32(base) + k.astype(np.float32) * step).astype(np.float32)
        d = float(x.max()) - float(x.min())
        with np.errstate(over="ignore"):
            assert np.isinf(np.float32(qmax) / np.float32(d))  # the formula as written overflows
        codes, s, z = orc.quantize_group(x, bits)
        assert s == step and z == np.float32(base)
        assert codes.tolist() == k.tolist()
        assert [orc.dequant(c, s, z) for c in codes] == x.tolist()


@pytest.mark.parametrize("bits", BITS)
def test_huge_range_progression_exact(orc, bits):
    """A span whose d = mx - mn overflows fp32: x_k = (2k - qmax) * 2^(128-bits),
    so d = 2^129 - 2^(129-bits) > FLT_MAX while every x_k is a finite bf16
    value.  Quantized at half size, code k comes out exactly, scale is
    2^(129-bits), zero = mn, and every x_k reconstructs exactly."""
    qmax = (1 << bits) - 1
    e = 128 - bits
    k = np.arange(qmax + 1)
    x = ((2 * k - qmax).astype(np.float64) * 2.0 ** e).astype(np.float32)
    assert np.all(np.isfinite(x)) and np.array_equal(bf16_round(x), x)
    with np.errstate(over="ignore"):
        assert np.isinf(np.float32(x.max()) - np.float32(x.min()))
    codes, s, z = orc.quantize_group(x, bits)
    assert s == np.float32(2.0 ** (e + 1)) and z == x.min()
    assert codes.tolist() == k.tolist()
    assert [orc.dequant(c, s, z) for c in codes] == x.tolist()


@pytest.mark.parametrize("bits", BITS)
def test_wide_ranges_match_fp64_quantizer(orc, bits):
    """Against the same quantizer evaluated in float64 (where neither range
    overflows): for groups of both extreme kinds the fp32 codes differ from
    the exact ones only where the fp64 value of (x - mn) * qmax / d lies
    within 1e-4 of a rounding boundary."""
    rng = np.random.default_rng(900 + bits)
    qmax = (1 << bits) - 1
    n = 0
    for x in random_groups(rng, 140, 64):
        x64 = x.astype(np.float64)
        d = x64.max() - x64.min()
        with np.errstate(over="ignore", divide="ignore"):
            wide = d > np.finfo(np.float32).max or np.isinf(np.float32(qmax) / np.float32(d))
        if not wide:
            continue
        n += 1
        codes, s, z = orc.quantize_group(x, bits)
        y = (x64 - x64.min()) * qmax / d
        exact = np.clip(np.rint(y), 0, qmax)
        frac = np.abs(y - np.floor(y) - 0.5)
        differ = codes != exact
        assert np.all(frac[differ] < 1e-4), (bits, y[differ], codes[differ])
        assert np.all(np.abs(codes.astype(np.int64) - exact) <= 1)
    assert n >= 20


def test_round_half_to_even(orc):
    """Exact half-way points round to the even code: with mn 0 and mx 3 at
    2 bits (scale 1), 0.5 -> 0, 1.5 -> 2, 2.5 -> 2."""
    x = np.array([0.0, 3.0, 0.5, 1.5, 2.5, 1.0], np.float32)
    codes, s, z = orc.quantize_group(x, 2)
    assert s == 1.0 and z == 0.0
    assert codes.tolist() == [0, 3, 0, 2, 2, 1]
    # 4 bits over [0, 15]: 6.5 -> 6, 7.5 -> 8
    x = np.array([0.0, 15.0, 6.5, 7.5, 14.5], np.float32)
    assert orc.quantize_group(x, 4)[0].tolist() == [0, 15, 6, 8, 14]


def test_no_fused_multiply_add(orc):
    """The code is round((x - mn) * inv) with both operations rounded.  Search
    inputs where a fused multiply-add, or a per-element division, would give a
    different code, and check the oracle picks the two-rounding answer."""
    rng = np.random.default_rng(7)
    hits = 0
    for _ in range(20000):
        x = bf16_round(rng.standard_normal(8).astype(np.float32) * np.float32(rng.uniform(0.1, 10)))
        mn, mx = np.float32(x.min()), np.float32(x.max())
        d = np.float32(mx - mn)
        if d == 0:
            continue
        qmax = np.float32(63)
        inv = np.float32(qmax / d)
        two = [np.float32(np.float32(xi - mn) * inv) for xi in x]
        exact = [float(xi - mn) * float(inv) for xi in x]   # the fused product, unrounded
        for i in range(8):
            a, b = np.rint(two[i]), np.rint(exact[i])
            if a != b:
                hits += 1
                codes, _, _ = orc.quantize_group(x, 6)
                assert codes[i] == int(a)
    assert hits > 0  # the search did reach the case it guards


# ---------------------------------------------------------------- compression

def test_compression_ratios_match_pages(orc):
    """Measured bytes of packed buffers vs bf16 reproduce the ratios the pages
    print (3.2x for K6V4, 2.56x for TurboQuant 6-bit) and the contract's
    figures (tests/golden/compression_ratios.txt)."""
    for line in open(os.path.join(GOLDEN, "compression_ratios.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        label, kb, vb, D, G, meta, want = [s.strip() for s in line.split("|")]
        kb, vb, D, G, meta, want = int(kb), int(vb), int(D), int(G), int(meta), float(want)
        B, H, T = 1, 1, 8
        x = W.bf16_bits(torch.randn(B, H, T, D).to(torch.bfloat16))
        sl = np.array([T], np.int32)
        cache = orc.quantize_kv(kb, vb if vb else kb, G, x, x, sl)
        n_t = 2 if vb else 1
        src = n_t * x.size * 2
        packed = cache["k_codes"].nbytes + (cache["v_codes"].nbytes if vb else 0)
        if meta:  # a 16-bit (passthrough) tensor has no (scale, zero)
            packed += (cache["k_sz"].nbytes if kb < 16 else 0) + (cache["v_sz"].nbytes if 0 < vb < 16 else 0)
        assert src / packed == pytest.approx(want, rel=1e-12), label


def test_passthrough_width_keeps_the_values(orc):
    """16 bits (Super KV Compression §第一层, outlier layers kept in 16-bit
    floating point): the row is the bf16 values themselves, byte for byte,
    with no (scale, zero) written, and reconstructs every value exactly --
    NaN and infinity included; K and V can take different widths."""
    rng = np.random.default_rng(3)
    B, H, T, D, G = 2, 2, 9, 64, 32
    x = rng.standard_normal((B, H, T, D)).astype(np.float32) * np.float32(100)
    x[0, 0, 0, :4] = [np.inf, -np.inf, np.nan, 3e38]
    kb16 = W.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    vb16 = W.bf16_bits(torch.from_numpy(-x).to(torch.bfloat16))
    sl = np.array([9, 4], np.int32)
    cache = orc.quantize_kv(16, 4, G, kb16, vb16, sl)
    assert orc.row_bytes(16, D) == 2 * D
    for b in range(B):
        n = int(sl[b])
        assert np.array_equal(cache["k_codes"][b, :, :n].reshape(-1), kb16[b, :, :n].reshape(-1).view(np.uint8))
        assert not cache["k_codes"][b, :, n:].any()
        kh = orc.dequant_rows(cache["k_codes"][b, :, :n].copy(), cache["k_sz"][b, :, :n].copy(), D, G, 16)
        want = torch.from_numpy(kb16[b, :, :n].view(np.int16)).view(torch.bfloat16).float().numpy()
        assert np.array_equal(kh.view(np.uint32), want.view(np.uint32))  # bit-exact, NaN included
    assert not cache["k_sz"].any()                 # nothing written for the 16-bit tensor
    assert cache["v_sz"][0, :, :9].any()          # the 4-bit tensor has its (scale, zero)


@pytest.mark.parametrize("kb,vb", [(16, 16), (16, 4), (6, 16)])
def test_decode_passthrough_vs_torch(orc, kb, vb):
    """Decode over caches with a 16-bit tensor against torch float64 softmax
    over the reconstructed values; K16V16 at tau 0 is plain attention over
    the bf16 cache."""
    cfg = W.scaled(W.CONFIGS[1], seed=70 + kb + vb)
    inp = W.make_inputs(cfg, seq_lens=torch.tensor([200], dtype=torch.int32))
    k, v, q, sl = (W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"]), W.bf16_bits(inp["q"]), inp["seq_lens"].numpy())
    cache = orc.quantize_kv(kb, vb, cfg.G, k, v, sl)
    kh, vh = _dequant_cache(orc, cache, kb, vb, cfg.D, cfg.G)
    for tau in (0.0, 1e-3):
        out, _, _ = orc.decode_attention(kb, vb, cfg.G, sl, q, cache, cfg.softmax_scale, tau)
        want = _torch_attention(q, kh, vh, sl, cfg.softmax_scale, tau)
        assert np.abs(out - want).max() <= 1e-6 * max(1.0, np.abs(want).max())
    if kb == vb == 16:
        bf = _torch_attention(q, _bf16_f32(k), _bf16_f32(v), sl, cfg.softmax_scale, 0.0)
        out, _, _ = orc.decode_attention(kb, vb, cfg.G, sl, q, cache, cfg.softmax_scale, 0.0)
        assert np.abs(out - bf).max() <= 1e-6


# ---------------------------------------------------------------- attention

def _dequant_cache(orc, cache, kb, vb, D, G):
    kh = orc.dequant_rows(cache["k_codes"], cache["k_sz"], D, G, kb)
    vh = orc.dequant_rows(cache["v_codes"], cache["v_sz"], D, G, vb)
    return kh, vh


def _torch_attention(q_bf16, kh, vh, seq_lens, scale, tau):
    """Independent reference: torch float64 softmax over the dequantized cache."""
    q = torch.from_numpy(q_bf16.view(np.int16)).view(torch.bfloat16).double()
    B, Hq, D = q.shape
    Hkv = kh.shape[1]
    r = Hq // Hkv
    out = torch.zeros(B, Hq, D, dtype=torch.float64)
    for b in range(B):
        T = int(seq_lens[b])
        if T == 0:
            continue
        K = torch.from_numpy(kh[b, :, :T]).double().repeat_interleave(r, dim=0)   # [Hq, T, D]
        V = torch.from_numpy(vh[b, :, :T]).double().repeat_interleave(r, dim=0)
        s = torch.einsum("hd,htd->ht", q[b], K) * float(np.float32(scale))
        p = torch.softmax(s, dim=-1)
        p = torch.where(p < float(np.float32(tau)), torch.zeros_like(p), p)
        out[b] = torch.einsum("ht,htd->hd", p, V)
    return out.numpy()


def _case(orc, cfg, kb, vb, seq_lens=None):
    inp = W.make_inputs(cfg, seq_lens=seq_lens)
    k, v, q, sl = (W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"]), W.bf16_bits(inp["q"]),
                   inp["seq_lens"].numpy())
    cache = orc.quantize_kv(kb, vb, cfg.G, k, v, sl)
    return q, cache, sl


@pytest.mark.parametrize("kb,vb", [(6, 4), (8, 8), (4, 2), (2, 6)])
def test_decode_matches_torch_fp64(orc, kb, vb):
    """Tiny inputs: the oracle equals torch float64 softmax attention over the
    dequantized cache to 1e-12 relative."""
    cfg = W.scaled(W.CONFIGS[1], seed=11 + kb)
    q, cache, sl = _case(orc, cfg, kb, vb)
    out, mask, counts = orc.decode_attention(kb, vb, cfg.G, sl, q, cache, cfg.softmax_scale, 0.0)
    kh, vh = _dequant_cache(orc, cache, kb, vb, cfg.D, cfg.G)
    ref = _torch_attention(q, kh, vh, sl, cfg.softmax_scale, 0.0)
    assert np.max(np.abs(out - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref))) + 1e-7 * np.max(np.abs(ref))
    assert mask.sum() == 0 and counts.tolist() == [0, 0]


def test_decode_ragged_and_gqa_vs_torch(orc):
    """Ragged lengths (including 0 and 1), GQA ratio 4, D 128, sparse-V skip."""
    cfg = W.scaled(W.CONFIGS[2], B=4, T_cap=96, seed=5)
    sl = torch.tensor([96, 1, 0, 37], dtype=torch.int32)
    q, cache, sl = _case(orc, cfg, 6, 4, seq_lens=sl)
    for tau in (0.0, 1e-3, 0.05):
        out, mask, counts = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, tau)
        kh, vh = _dequant_cache(orc, cache, 6, 4, cfg.D, cfg.G)
        ref = _torch_attention(q, kh, vh, sl, cfg.softmax_scale, tau)
        np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-6)
        assert np.all(out[2] == 0.0)        # empty sequence attends to nothing
        assert counts[0] == int(mask.sum())


def test_q_zero_gives_mean_of_v(orc):
    """q = 0 and tau = 0: every probability is 1/T, so out = mean_t vhat_t."""
    cfg = W.CONFIGS[1]
    q, cache, sl = _case(orc, cfg, 6, 4)
    q = np.zeros_like(q)
    out, _, _ = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, 0.0)
    vh = orc.dequant_rows(cache["v_codes"], cache["v_sz"], cfg.D, cfg.G, 4).astype(np.float64)
    want = vh[0, :, : sl[0]].mean(axis=1)                       # [Hkv, D]
    want = np.repeat(want, cfg.r, axis=0).astype(np.float32)
    np.testing.assert_allclose(out[0], want, rtol=0, atol=2e-7 * np.abs(vh).max())


def test_one_hot_heavy_hitter_returns_its_v(orc):
    """One key whose logit beats every other by >= 60 returns its V row; with
    tau > 0 every other row is skipped."""
    D, T, G = 64, 40, 32
    rng = np.random.default_rng(3)
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, :] = 1.0
    k = np.zeros((1, 1, T, D), np.float32)
    k[0, 0] = bf16_round(rng.uniform(-0.5, 0.5, (T, D)))
    t_star = 17
    k[0, 0, t_star] = 16.0                       # logit 64*16/8 = 128 vs <= 2
    v = bf16_round(rng.standard_normal((1, 1, T, D)))
    kbits = W.bf16_bits(torch.from_numpy(k).to(torch.bfloat16))
    vbits = W.bf16_bits(torch.from_numpy(v).to(torch.bfloat16))
    qbits = W.bf16_bits(torch.from_numpy(q).to(torch.bfloat16))
    sl = np.array([T], np.int32)
    cache = orc.quantize_kv(6, 4, G, kbits, vbits, sl)
    vh = orc.dequant_rows(cache["v_codes"], cache["v_sz"], D, G, 4)
    for tau in (0.0, 1e-6):
        out, mask, counts = orc.decode_attention(6, 4, G, sl, qbits, cache, 0.125, tau)
        np.testing.assert_allclose(out[0, 0], vh[0, 0, t_star], rtol=1e-6, atol=1e-7)
        if tau > 0:
            assert mask[0, 0].sum() == T - 1 and mask[0, 0, t_star] == 0
            assert counts.tolist() == [T - 1, T - 1]


def test_tau_special_cases(orc):
    """tau = 0 skips nothing and equals dense attention; tau above every
    probability skips everything and gives zeros (no renormalisation)."""
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=64, seed=9)
    q, cache, sl = _case(orc, cfg, 6, 4)
    dense, m0, c0 = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, 0.0)
    assert m0.sum() == 0 and c0.tolist() == [0, 0]
    out, m1, c1 = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, 1.01)
    assert np.all(out == 0.0)
    assert c1.tolist() == [cfg.B * cfg.Hq * 64, cfg.B * cfg.Hkv * 64]
    # skipped mass is dropped, not renormalised: out(tau) = dense - sum of skipped p*v
    kh, vh = _dequant_cache(orc, cache, 6, 4, cfg.D, cfg.G)
    ref = _torch_attention(q, kh, vh, sl, cfg.softmax_scale, 0.02)
    out, m2, _ = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, 0.02)
    assert 0 < m2.sum() < m2.size
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-7)
    assert np.linalg.norm(out - dense) > 1e-4


def test_skip_set_matches_torch_probabilities(orc):
    """The skip mask is exactly {p < tau} for float64 probabilities from torch,
    outside a 1e-7 band around tau."""
    cfg = W.scaled(W.CONFIGS[2], B=1, T_cap=512, seed=21)
    q, cache, sl = _case(orc, cfg, 6, 4)
    tau = 1e-3
    _, mask, counts = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, tau)
    kh, _ = _dequant_cache(orc, cache, 6, 4, cfg.D, cfg.G)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()[0]
    K = torch.from_numpy(kh[0]).double().repeat_interleave(cfg.r, dim=0)
    p = torch.softmax(torch.einsum("hd,htd->ht", qd, K) * float(np.float32(cfg.softmax_scale)), -1).numpy()
    want = p < float(np.float32(tau))
    band = np.abs(p - tau) < 1e-7
    assert np.all((mask[0] == 1) == want | band) and np.all((mask[0] == 1) | ~want | band)
    rows_all = (mask[0].reshape(cfg.Hkv, cfg.r, -1).min(axis=1) == 1).sum()
    assert counts.tolist() == [int(mask.sum()), int(rows_all)]


def test_attention_mass_is_group_mean_of_torch_softmax(orc):
    """The per-token mass fed to the next step's tiers is the mean over the
    group's query heads of torch float64 softmax probabilities; over t it
    sums to 1 per (b, KV head); slots beyond T_b stay 0; with one query head
    per group it is that head's probability."""
    cfg = W.scaled(W.CONFIGS[2], B=2, T_cap=384, seed=23)
    q, cache, sl = _case(orc, cfg, 6, 4)
    sl = np.array([384, 200], np.int32)
    _, _, _, p = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, 1e-3, want_p=True)
    mass = orc.attention_mass(p, cfg.Hkv, sl)
    kh, _ = _dequant_cache(orc, cache, 6, 4, cfg.D, cfg.G)
    for b in range(2):
        T = int(sl[b])
        qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()[b]
        K = torch.from_numpy(kh[b, :, :T]).double().repeat_interleave(cfg.r, dim=0)
        pt = torch.softmax(torch.einsum("hd,htd->ht", qd, K) * float(np.float32(cfg.softmax_scale)), -1).numpy()
        want = pt.reshape(cfg.Hkv, cfg.r, T).mean(axis=1)
        np.testing.assert_allclose(mass[b, :, :T], want, rtol=1e-9, atol=1e-15)
        np.testing.assert_allclose(mass[b, :, :T].sum(axis=1), 1.0, rtol=1e-12)
        assert np.all(mass[b, :, T:] == 0.0)
    one = orc.attention_mass(p[:, ::cfg.r], cfg.Hkv, sl)      # one head per group
    np.testing.assert_array_equal(one, p[:, ::cfg.r])


# ---------------------------------------------------------------- tiers

# ---------------------------------------------------------------- bf16-cache attention

def _bf16_f32(a_bits):
    return torch.from_numpy(np.ascontiguousarray(a_bits).view(np.int16)).view(torch.bfloat16).float().numpy()


def test_attention_bf16_vs_torch_fp64(orc):
    """The unquantized-cache attention (the reference the quantized decode's
    quality is measured against) matches torch float64 softmax over the same
    bf16 values, ragged lengths and GQA included, T = 0 giving zeros."""
    cfg = W.scaled(W.CONFIGS[4], B=5, T_cap=150, seq_lo=1, seq_hi=150, seed=31)
    inp = W.make_inputs(cfg, seq_lens=torch.tensor([150, 1, 0, 77, 149], dtype=torch.int32))
    k, v, q, sl = (W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"]), W.bf16_bits(inp["q"]), inp["seq_lens"].numpy())
    got = orc.attention_bf16(sl, q, k, v, cfg.softmax_scale)
    want = _torch_attention(q, _bf16_f32(k), _bf16_f32(v), sl, cfg.softmax_scale, 0.0)
    assert np.abs(got - want).max() <= 1e-6 * max(1.0, np.abs(want).max())
    assert np.all(got[2] == 0)
    # T = 1: the output is that row's V exactly (p = 1)
    r = cfg.Hq // cfg.Hkv
    assert np.array_equal(got[1], np.repeat(_bf16_f32(v)[1, :, 0], r, axis=0))


def test_attention_bf16_closed_forms(orc):
    """q = 0 gives the mean of V; a key far along q returns its V row."""
    B, Hq, Hkv, T, D = 1, 4, 2, 33, 64
    rng = np.random.default_rng(5)
    v = bf16_round(rng.standard_normal((B, Hkv, T, D)).astype(np.float32))
    k = bf16_round(rng.standard_normal((B, Hkv, T, D)).astype(np.float32))
    tob = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    sl = np.array([T], np.int32)
    out = orc.attention_bf16(sl, tob(np.zeros((B, Hq, D))), tob(k), tob(v), 0.125)
    mean = v.astype(np.float64).mean(axis=2)
    assert np.abs(out[0] - np.repeat(mean[0], 2, axis=0)).max() <= 1e-6
    q = bf16_round(rng.standard_normal((B, Hq, D)).astype(np.float32))
    k2 = k.copy()
    k2[0, 1, 7] = bf16_round(q[0, 2] * 40)   # KV head 1 serves query heads 2 and 3
    out = orc.attention_bf16(sl, tob(q), tob(k2), tob(v), 1.0)
    assert np.abs(out[0, 2] - v[0, 1, 7]).max() <= 1e-6


def test_tier_boundaries(orc):
    """Super KV Compression §第二层: above tau_high -> 6-bit V (2), within
    [tau_low, tau_high] -> 4-bit V (1), below tau_low -> evicted (0)."""
    lo, hi = np.float32(1e-4), np.float32(1e-2)
    vals = [hi, np.nextafter(hi, np.float32(1)), lo, np.nextafter(lo, np.float32(0)),
            np.float32(0.5), np.float32(0.0), np.float32(np.nan), np.float32(3e-3)]
    want = [1, 2, 1, 0, 2, 0, 0, 1]
    T_cap = 12
    mass = np.zeros((1, 1, T_cap), np.float32)
    mass[0, 0, : len(vals)] = vals
    mass[0, 0, len(vals):] = 0.9                          # beyond T_b: ignored
    tier, counts, p2, p1 = orc.tier_classify(np.array([len(vals)], np.int32), mass, lo, hi)
    assert tier[0, 0].tolist() == want + [0] * (T_cap - len(vals))
    assert counts[0, 0].tolist() == [2, 3]
    assert p2[0, 0, :2].tolist() == [1, 4]
    assert p1[0, 0, :3].tolist() == [0, 2, 7]


def test_tier_positions_complete_and_sorted(orc):
    cfg = W.scaled(W.CONFIGS[5], B=3, T_cap=2048, seq_lo=100, seq_hi=2048, seed=13)
    inp = W.make_inputs(cfg, with_mass=True)
    sl, mass = inp["seq_lens"].numpy(), inp["mass"].numpy()
    tier, counts, p2, p1 = orc.tier_classify(sl, mass, cfg.tau_low, cfg.tau_high)
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            T = sl[b]
            a = mass[b, g, :T]
            hi_pos = np.nonzero(a > np.float32(cfg.tau_high))[0]
            mid_pos = np.nonzero((a >= np.float32(cfg.tau_low)) & (a <= np.float32(cfg.tau_high)))[0]
            assert counts[b, g].tolist() == [hi_pos.size, mid_pos.size]
            assert p2[b, g, : hi_pos.size].tolist() == hi_pos.tolist()
            assert p1[b, g, : mid_pos.size].tolist() == mid_pos.tolist()
            assert np.all(tier[b, g, T:] == 0)


def test_tier_repack_rows_within_bound(orc):
    """Each kept token is re-quantized from bf16 at its tier's width: K6 in
    both segments, V6 in A and V4 in B, within the quantizer's error bound."""
    cfg = W.scaled(W.CONFIGS[5], B=2, T_cap=1024, seq_lo=1024, seq_hi=1024, seed=17)
    inp = W.make_inputs(cfg, with_mass=True)
    k, v = W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"])
    sl, mass = inp["seq_lens"].numpy(), inp["mass"].numpy()
    _, counts, p2, p1 = orc.tier_classify(sl, mass, cfg.tau_low, cfg.tau_high)
    A, Bs = orc.tier_repack(cfg.G, k, v, counts, p2, p1)
    kf, vf = inp["k"].float().numpy(), inp["v"].float().numpy()
    for seg, pos, vbits, n_i in ((A, p2, 6, 0), (Bs, p1, 4, 1)):
        kh = orc.dequant_rows(seg["k_codes"], seg["k_sz"], cfg.D, cfg.G, 6)
        vh = orc.dequant_rows(seg["v_codes"], seg["v_sz"], cfg.D, cfg.G, vbits)
        for b in range(cfg.B):
            for g in range(cfg.Hkv):
                n = counts[b, g, n_i]
                assert n > 0
                src = pos[b, g, :n]
                for xh, x, sz in ((kh, kf, seg["k_sz"]), (vh, vf, seg["v_sz"])):
                    err = np.abs(xh[b, g, :n] - x[b, g, src]).reshape(n, -1, cfg.G)
                    scale = sz[b, g, :n, :, 0][..., None]
                    assert np.all(err <= scale / 2 + 2 * np.spacing(np.abs(x[b, g, src]).max()))


def test_tiered_attention_vs_torch_and_plain(orc):
    """One softmax over the kept tokens of both segments equals torch float64
    attention over those rows; with tau_low = 0 and tau_high = inf every token
    lands in segment B and the result equals plain K6V4 decode."""
    cfg = W.scaled(W.CONFIGS[5], B=2, T_cap=1500, seq_lo=700, seq_hi=1500, seed=19)
    inp = W.make_inputs(cfg, with_mass=True)
    k, v, q = W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"]), W.bf16_bits(inp["q"])
    sl, mass = inp["seq_lens"].numpy(), inp["mass"].numpy()
    tier, counts, p2, p1 = orc.tier_classify(sl, mass, cfg.tau_low, cfg.tau_high)
    A, Bs = orc.tier_repack(cfg.G, k, v, counts, p2, p1)
    out, _ = orc.tiered_attention(cfg.G, counts, q, A, Bs, cfg.softmax_scale, 0.0)
    # independent: gather kept rows, dequantize, torch softmax
    akh = orc.dequant_rows(A["k_codes"], A["k_sz"], cfg.D, cfg.G, 6)
    avh = orc.dequant_rows(A["v_codes"], A["v_sz"], cfg.D, cfg.G, 6)
    bkh = orc.dequant_rows(Bs["k_codes"], Bs["k_sz"], cfg.D, cfg.G, 6)
    bvh = orc.dequant_rows(Bs["v_codes"], Bs["v_sz"], cfg.D, cfg.G, 4)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            g = h // cfg.r
            na, nb = counts[b, g]
            K = np.concatenate([akh[b, g, :na], bkh[b, g, :nb]]).astype(np.float64)
            V = np.concatenate([avh[b, g, :na], bvh[b, g, :nb]]).astype(np.float64)
            p = torch.softmax(torch.from_numpy(K) @ qd[b, h] * float(np.float32(cfg.softmax_scale)), 0)
            ref = (p[:, None] * torch.from_numpy(V)).sum(0).numpy()
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-6, atol=1e-7)
    # all tokens kept at 4-bit V == plain K6V4 decode
    tier, counts, p2, p1 = orc.tier_classify(sl, mass, 0.0, np.inf)
    assert np.all(counts[..., 0] == 0) and np.all(counts[..., 1] == sl[:, None])
    A, Bs = orc.tier_repack(cfg.G, k, v, counts, p2, p1)
    out_t, _ = orc.tiered_attention(cfg.G, counts, q, A, Bs, cfg.softmax_scale, 0.0)
    cache = orc.quantize_kv(6, 4, cfg.G, k, v, sl)
    out_p, _, _ = orc.decode_attention(6, 4, cfg.G, sl, q, cache, cfg.softmax_scale, 0.0)
    np.testing.assert_array_equal(out_t, out_p)
