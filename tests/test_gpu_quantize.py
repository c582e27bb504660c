"""lkv_quantize_kv on the GPU vs the CPU oracle: packed codes and (scale,
zero) must be bit-exact ("Super KV Compression" §第一层, "TurboQuant"
§TurboQuant的核心创新)."""
import numpy as np
import pytest
import torch

from gpu_helpers import gpu_quantize, oracle_inputs
from quantized_kv_cache_lkv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def compare_cache(gpu, want, seq_lens, what):
    sl = np.asarray(seq_lens)
    for key in ("k_codes", "k_sz", "v_codes", "v_sz"):
        g = gpu[key].cpu().numpy()
        w = want[key]
        for b in range(g.shape[0]):
            T = int(sl[b])
            gb, wb = g[b, :, :T], w[b, :, :T]
            if key.endswith("sz"):
                gb, wb = gb.view(np.uint32), wb.view(np.uint32)
            if not np.array_equal(gb, wb):
                n = int((gb != wb).sum())
                raise AssertionError(f"{what} {key} b={b}: {n} entries differ")


def special_rows(inp):
    """Overwrite a few rows with degenerate groups: constants, zeros of both
    signs, a single outlier, huge and tiny magnitudes."""
    k, v = inp["k"], inp["v"]
    D = k.shape[-1]
    k[0, 0, 0] = 0.0
    v[0, 0, 0] = -0.0
    k[0, 0, 1] = 3.5
    v[0, 0, 1, : D // 2] = -0.0
    v[0, 0, 1, D // 2:] = 0.0
    k[0, 0, 2] = torch.linspace(-1e30, 1e30, D).to(torch.bfloat16)
    v[0, 0, 2] = torch.linspace(-1e-30, 1e-30, D).to(torch.bfloat16)
    k[0, 0, 3] = 1.0
    k[0, 0, 3, 5] = 1000.0
    v[0, 0, 3] = torch.arange(D, dtype=torch.float32).remainder(16).to(torch.bfloat16)
    # range so small that qmax / d overflows (subnormal steps), and so large
    # that d = mx - mn overflows: both take the clamped path of the formula
    v[0, 0, 4] = torch.linspace(0.0, 1e-38, 16, dtype=torch.float64).repeat(D // 16).to(torch.bfloat16)
    k[0, 0, 4] = torch.linspace(-3e38, 3e38, 16, dtype=torch.float64).repeat(D // 16).to(torch.bfloat16)
    # random spans of +-1e38..3e38, random subnormal values, and a few
    # near-subnormal steps around 2^-120
    g = torch.Generator().manual_seed(D)
    k[0, 0, 5] = ((torch.rand(D, generator=g, dtype=torch.float64) * 6 - 3) * 1e38).to(torch.bfloat16)
    v[0, 0, 5] = (torch.randn(D, generator=g, dtype=torch.float64) * 1e-39).to(torch.bfloat16)
    k[0, 0, 6] = (2.0 ** -120 + torch.randint(-2, 3, (D,), generator=g).double() * 2.0 ** -127).to(torch.bfloat16)
    v[0, 0, 6] = ((torch.rand(D, generator=g, dtype=torch.float64) * 2 + 1) * 1e38).to(torch.bfloat16)
    v[0, 0, 6, ::3] *= -1
    return inp


@pytest.mark.parametrize("D,G", [(64, 32), (64, 64), (128, 32), (128, 64), (128, 128)])
@pytest.mark.parametrize("kb,vb", [(6, 4), (8, 8), (4, 4), (4, 2), (2, 8), (8, 6), (2, 2), (6, 6),
                                   (16, 4), (6, 16), (16, 16)])
def test_quantize_bit_exact_small(orc, D, G, kb, vb):
    cfg = W.Config("q", B=3, Hq=4, Hkv=2, D=D, T_cap=80, G=G, bits=[(kb, vb)], seed=D + G + kb * 7 + vb)
    inp = special_rows(W.make_inputs(cfg, seq_lens=torch.tensor([80, 37, 0], dtype=torch.int32)))
    gpu = gpu_quantize(kb, vb, G, inp)
    k, v, _, sl = oracle_inputs(inp)
    want = orc.quantize_kv(kb, vb, G, k, v, sl)
    compare_cache(gpu, want, sl, f"K{kb}V{vb} D{D} G{G}")
    # rows beyond the sequence length stay untouched (zero-filled here)
    assert int(gpu["k_codes"][1, :, 37:].abs().sum()) == 0 and int(gpu["v_sz"][2].abs().sum()) == 0


def test_quantize_config1_tiny(orc):
    cfg = W.CONFIGS[1]
    inp = W.make_inputs(cfg)
    gpu = gpu_quantize(6, 4, cfg.G, inp)
    k, v, _, sl = oracle_inputs(inp)
    compare_cache(gpu, orc.quantize_kv(6, 4, cfg.G, k, v, sl), sl, "config 1")


def test_quantize_long_context_full_size_sampled(orc):
    """The 131072-token K/V of the long-context workload quantized in one
    launch; the oracle checks the first, a middle and the last 2048 rows of
    every KV head."""
    cfg = W.CONFIGS[3]
    inp = W.make_inputs(cfg)
    gpu = gpu_quantize(6, 4, cfg.G, inp)
    T = cfg.T_cap
    for t0 in (0, T // 2 - 1000, T - 2048):
        sub = {"k": inp["k"][:, :, t0:t0 + 2048].contiguous(), "v": inp["v"][:, :, t0:t0 + 2048].contiguous()}
        sl = np.array([2048], np.int32)
        want = orc.quantize_kv(6, 4, cfg.G, W.bf16_bits(sub["k"]), W.bf16_bits(sub["v"]), sl)
        got = {k: v[:, :, t0:t0 + 2048] for k, v in gpu.items()}
        compare_cache(got, want, sl, f"config 3 rows {t0}..")


def test_quantize_out_of_range_lengths_are_clamped(orc):
    cfg = W.Config("q", B=2, Hq=4, Hkv=2, D=64, T_cap=32, G=32, bits=[(6, 4)], seed=3)
    inp = W.make_inputs(cfg)
    inp["seq_lens"] = torch.tensor([999, -5], dtype=torch.int32)
    gpu = gpu_quantize(6, 4, 32, inp)
    k, v, _, _ = oracle_inputs(inp)
    want = orc.quantize_kv(6, 4, 32, k, v, np.array([32, 0], np.int32))
    compare_cache(gpu, want, [32, 0], "clamped")
    assert int(gpu["k_codes"][1].abs().sum()) == 0


@pytest.mark.parametrize("D,G,kb,vb", [(128, 64, 6, 4), (64, 32, 8, 8), (128, 128, 4, 2), (128, 32, 2, 6),
                                       (128, 64, 16, 4), (64, 32, 16, 16)])
def test_append_equals_quantize_of_the_longer_sequence(orc, D, G, kb, vb):
    """lkv_append_kv writes the new token's row exactly as lkv_quantize_kv
    would (bit-exact vs the oracle), and touches no other row; positions
    outside [0, T_cap) write nothing."""
    from quantized_kv_cache_lkv_b200 import lkv
    T_cap = 96
    cfg = W.Config("append", B=4, Hq=4, Hkv=2, D=D, T_cap=T_cap, G=G, bits=[(kb, vb)], seed=90 + D + G + kb)
    full = torch.tensor([50, 96, 1, 20], dtype=torch.int32)
    inp = W.make_inputs(cfg, seq_lens=full)
    # two appended rows carry the extreme ranges: a span whose d overflows fp32
    # and subnormal values whose qmax / d overflows
    g = torch.Generator().manual_seed(D + kb)
    inp["k"][0, :, 49] = ((torch.rand(2, D, generator=g, dtype=torch.float64) * 6 - 3) * 1e38).to(torch.bfloat16)
    inp["v"][1, :, 95] = (torch.randn(2, D, generator=g, dtype=torch.float64) * 1e-39).to(torch.bfloat16)
    before = torch.tensor([49, 95, 0, 20], dtype=torch.int32)   # sequence 3 appends at an invalid slot below
    cache = gpu_quantize(kb, vb, G, dict(inp, seq_lens=before))
    pos = torch.tensor([49, 95, 0, T_cap], dtype=torch.int32)    # T_cap: nothing written
    k_new = torch.stack([inp["k"][b, :, min(int(pos[b]), T_cap - 1)] for b in range(4)]).contiguous()
    v_new = torch.stack([inp["v"][b, :, min(int(pos[b]), T_cap - 1)] for b in range(4)]).contiguous()
    snapshot = {k: v.clone() for k, v in cache.items()}
    lkv.lkv_append_kv((kb, vb, G), 4, 2, T_cap, D, pos.cuda(), k_new.cuda(), v_new.cuda(), cache["k_codes"],
                      cache["k_sz"], cache["v_codes"], cache["v_sz"])
    torch.cuda.synchronize()
    after = torch.tensor([50, 96, 1, 20], dtype=torch.int32)
    k, v, _, sl = oracle_inputs(dict(inp, seq_lens=after))
    want = orc.quantize_kv(kb, vb, G, k, v, sl)
    compare_cache(cache, want, sl, f"append K{kb}V{vb} D{D} G{G}")
    for key in cache:   # rows other than the appended ones are untouched
        g, s0 = cache[key].cpu(), snapshot[key].cpu()
        for b in range(4):
            keep = [t for t in range(T_cap) if not (b < 3 and t == int(pos[b]))]
            assert torch.equal(g[b, :, keep], s0[b, :, keep]), (key, b)


@pytest.mark.parametrize("kb,vb", [(16, 16), (16, 4), (6, 16)])
def test_passthrough_width_rows_are_the_bf16_values(kb, vb):
    """At 16 bits the cache row is the bf16 row itself, byte for byte, and
    the (scale, zero) of that tensor is never written (it may be omitted)."""
    from quantized_kv_cache_lkv_b200 import buffers, lkv
    from gpu_helpers import dev
    cfg = W.Config("pass", B=2, Hq=4, Hkv=2, D=128, T_cap=64, G=64, bits=[(kb, vb)], seed=8)
    inp = W.make_inputs(cfg, seq_lens=torch.tensor([64, 10], dtype=torch.int32))
    cache = buffers.alloc_cache(kb, vb, 64, 2, 2, 64, 128, zero=True)
    lkv.lkv_quantize_kv((kb, vb, 64), 2, 2, 64, 128, dev(inp["seq_lens"]), dev(inp["k"]), dev(inp["v"]),
                        cache["k_codes"], None if kb == 16 else cache["k_sz"], cache["v_codes"],
                        None if vb == 16 else cache["v_sz"])
    torch.cuda.synchronize()
    for bits, key, src in ((kb, "k", inp["k"]), (vb, "v", inp["v"])):
        if bits != 16:
            continue
        got = cache[key + "_codes"].cpu()
        for b, T in enumerate((64, 10)):
            assert torch.equal(got[b, :, :T].view(torch.bfloat16), src[b, :, :T])
            assert int(got[b, :, T:].abs().sum()) == 0
        assert int(cache[key + "_sz"].abs().sum()) == 0
