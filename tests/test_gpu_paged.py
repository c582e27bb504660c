"""Paged caches: the pool-and-block-table calls give exactly what the
contiguous calls give on the same tokens, and what the CPU oracle gives,
with the pages scattered over a pool in random order ("TurboQuant" §与其他优化技术的对比: the quantized
cache is meant to combine with paged KV management)."""
import numpy as np
import pytest
import torch

from gpu_helpers import (assert_attention_close, assert_masks_match, dev, gpu_decode, gpu_quantize, oracle_inputs,
                         vmax)
from quantized_kv_cache_lkv_b200 import buffers, lkv
from quantized_kv_cache_lkv_b200 import workloads as W

pytestmark = pytest.mark.gpu
P = lkv.LKV_PAGE_TOKENS


def make_pool(kb, vb, G, Hkv, D, num_pages):
    ng = D // G
    return {"k_codes": torch.zeros(num_pages, Hkv, P, D * kb // 8, dtype=torch.uint8, device="cuda"),
            "k_sz": torch.zeros(num_pages, Hkv, P, ng, 2, device="cuda"),
            "v_codes": torch.zeros(num_pages, Hkv, P, D * vb // 8, dtype=torch.uint8, device="cuda"),
            "v_sz": torch.zeros(num_pages, Hkv, P, ng, 2, device="cuda")}


def gather_pool(pool, table, B, T_cap):
    """The pool read back through the block table as [B][Hkv][T_cap][...]."""
    out = {}
    for key, t in pool.items():
        rows = [torch.cat([t[int(table[b, i])] for i in range(table.shape[1])], dim=1) for b in range(B)]
        out[key] = torch.stack(rows)[:, :, :T_cap]
    return out


def setup(kb=6, vb=4, G=64, r=4, seed=3, lens=(768, 300, 1)):
    B, Hkv, D, pps = len(lens), 2, 128, 3
    T_cap = pps * P
    cfg = W.Config("paged", B=B, Hq=Hkv * r, Hkv=Hkv, D=D, T_cap=T_cap, G=G, bits=[(kb, vb)], hh_frac=0.01,
                   seed=seed)
    inp = W.make_inputs(cfg, seq_lens=torch.tensor(lens, dtype=torch.int32))
    num_pages = B * pps + 2
    gen = torch.Generator().manual_seed(seed)
    table = torch.randperm(num_pages, generator=gen)[:B * pps].view(B, pps).to(torch.int32)
    pool = make_pool(kb, vb, G, Hkv, D, num_pages)
    lkv.lkv_quantize_kv_paged((kb, vb, G), B, Hkv, pps, num_pages, D, dev(inp["seq_lens"]), dev(inp["k"]),
                              dev(inp["v"]), dev(table), pool["k_codes"], pool["k_sz"], pool["v_codes"],
                              pool["v_sz"])
    torch.cuda.synchronize()
    return cfg, inp, table, pool, num_pages


@pytest.mark.parametrize("kb,vb,G", [(6, 4, 64), (8, 8, 32), (4, 2, 128)])
def test_paged_quantize_equals_contiguous(orc, kb, vb, G):
    cfg, inp, table, pool, _ = setup(kb, vb, G)
    want = gpu_quantize(kb, vb, G, inp)
    got = gather_pool(pool, table, cfg.B, cfg.T_cap)
    k, v, _, sl = oracle_inputs(inp)
    o = orc.quantize_kv(kb, vb, G, k, v, sl)
    for key in want:
        for b in range(cfg.B):
            T = int(inp["seq_lens"][b])
            assert torch.equal(got[key][b, :, :T], want[key][b, :, :T]), (key, b)
            g = np.ascontiguousarray(got[key][b, :, :T].cpu().numpy())
            assert np.array_equal(g.view(np.uint8), np.ascontiguousarray(o[key][b, :, :T]).view(np.uint8)), (key, b)


@pytest.mark.parametrize("r,tau", [(4, 1e-3), (2, 0.0), (1, 1e-4)])
def test_paged_decode_equals_contiguous(orc, r, tau):
    """Same work partition, same arithmetic: outputs, masks and counts are
    bit-identical to the contiguous decode, and match the oracle."""
    cfg, inp, table, pool, num_pages = setup(r=r, seed=10 + r)
    cache = gpu_quantize(6, 4, 64, inp)
    want_out, want_mask, want_counts = gpu_decode(6, 4, 64, inp, cache, cfg.softmax_scale, tau)
    B, Hq, Hkv, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.D
    nb = lkv.lkv_decode_workspace_bytes((6, 4, 64), B, Hq, Hkv, cfg.T_cap, D)
    ws = buffers.alloc_workspace(nb)
    out = torch.empty(B, Hq, D, device="cuda")
    mask = torch.zeros(B, Hq, cfg.T_cap, dtype=torch.uint8, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    lkv.lkv_decode_attention_paged((6, 4, 64), B, Hq, Hkv, 3, num_pages, D, dev(inp["seq_lens"]), dev(inp["q"]),
                                   dev(table), pool["k_codes"], pool["k_sz"], pool["v_codes"], pool["v_sz"],
                                   cfg.softmax_scale, tau, out, mask, counts, ws, nb)
    torch.cuda.synchronize()
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_OK
    np.testing.assert_array_equal(out.cpu().numpy(), want_out)
    np.testing.assert_array_equal(mask.cpu().numpy(), want_mask)
    assert counts.cpu().tolist() == want_counts.tolist()
    k, v, q, sl = oracle_inputs(inp)
    o_out, o_mask, o_counts, p = orc.decode_attention(6, 4, 64, sl, q, orc.quantize_kv(6, 4, 64, k, v, sl),
                                                      cfg.softmax_scale, tau, want_p=True)
    assert_attention_close(out.cpu().numpy(), o_out, vmax(inp), "paged vs oracle")
    if assert_masks_match(mask.cpu().numpy(), o_mask, p, np.float32(tau), sl, "paged vs oracle") == 0:
        assert counts.cpu().tolist() == o_counts.tolist()


def test_paged_append_equals_contiguous(orc):
    cfg, inp, table, pool, num_pages = setup(lens=(767, 299, 0))
    pos = torch.tensor([767, 299, 0], dtype=torch.int32)
    k_new = torch.stack([inp["k"][b, :, int(pos[b])] for b in range(3)]).contiguous()
    v_new = torch.stack([inp["v"][b, :, int(pos[b])] for b in range(3)]).contiguous()
    lkv.lkv_append_kv_paged((6, 4, 64), 3, 2, 3, num_pages, 128, dev(pos), dev(k_new), dev(v_new), dev(table),
                            pool["k_codes"], pool["k_sz"], pool["v_codes"], pool["v_sz"])
    torch.cuda.synchronize()
    full = dict(inp, seq_lens=torch.tensor([768, 300, 1], dtype=torch.int32))
    want = gpu_quantize(6, 4, 64, full)
    got = gather_pool(pool, table, 3, cfg.T_cap)
    k, v, _, sl = oracle_inputs(full)
    o = orc.quantize_kv(6, 4, 64, k, v, sl)
    for key in want:
        for b in range(3):
            T = int(full["seq_lens"][b])
            assert torch.equal(got[key][b, :, :T], want[key][b, :, :T]), (key, b)
            g = np.ascontiguousarray(got[key][b, :, :T].cpu().numpy())
            assert np.array_equal(g.view(np.uint8), np.ascontiguousarray(o[key][b, :, :T]).view(np.uint8)), (key, b)


def test_paged_decode_bad_page_is_reported():
    """A page id outside the pool is read as page 0 and reported in the
    status word; the call does not fault and its outputs stay finite."""
    cfg, inp, table, pool, num_pages = setup()
    bad = table.clone()
    bad[1, 0] = num_pages + 5
    B, Hq, Hkv, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.D
    nb = lkv.lkv_decode_workspace_bytes((6, 4, 64), B, Hq, Hkv, cfg.T_cap, D)
    ws = buffers.alloc_workspace(nb)
    out = torch.empty(B, Hq, D, device="cuda")
    lkv.lkv_decode_attention_paged((6, 4, 64), B, Hq, Hkv, 3, num_pages, D, dev(inp["seq_lens"]), dev(inp["q"]),
                                   dev(bad), pool["k_codes"], pool["k_sz"], pool["v_codes"], pool["v_sz"],
                                   cfg.softmax_scale, 1e-3, out, None, None, ws, nb)
    torch.cuda.synchronize()
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_ERR_INVALID_ARG
    assert torch.isfinite(out).all()


@pytest.mark.slow
def test_paged_decode_full_size_equals_contiguous(orc):
    """The Llama-3.1-8B-shaped decode (B16, 32 q / 8 kv heads, T8192 = 32
    pages per sequence, tau 1e-4) over a shuffled pool of 520 pages is
    bit-identical to the contiguous decode, and every sequence matches the
    oracle."""
    cfg = W.CONFIGS[2]
    B, Hq, Hkv, D, T, G = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.T_cap, cfg.G
    pps = T // P
    inp = W.make_inputs(cfg)
    num_pages = B * pps + 8
    table = torch.randperm(num_pages, generator=torch.Generator().manual_seed(5))[:B * pps].view(B, pps)
    table = table.to(torch.int32)
    pool = make_pool(6, 4, G, Hkv, D, num_pages)
    sl = dev(inp["seq_lens"])
    lkv.lkv_quantize_kv_paged((6, 4, G), B, Hkv, pps, num_pages, D, sl, dev(inp["k"]), dev(inp["v"]), dev(table),
                              pool["k_codes"], pool["k_sz"], pool["v_codes"], pool["v_sz"])
    cache = gpu_quantize(6, 4, G, inp)
    want_out, want_mask, want_counts = gpu_decode(6, 4, G, inp, cache, cfg.softmax_scale, cfg.tau, want_mask=False)
    nb = lkv.lkv_decode_workspace_bytes((6, 4, G), B, Hq, Hkv, T, D)
    ws = buffers.alloc_workspace(nb)
    out = torch.empty(B, Hq, D, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    lkv.lkv_decode_attention_paged((6, 4, G), B, Hq, Hkv, pps, num_pages, D, sl, dev(inp["q"]), dev(table),
                                   pool["k_codes"], pool["k_sz"], pool["v_codes"], pool["v_sz"], cfg.softmax_scale,
                                   cfg.tau, out, None, counts, ws, nb)
    torch.cuda.synchronize()
    assert lkv.lkv_workspace_status(ws) == lkv.LKV_OK
    np.testing.assert_array_equal(out.cpu().numpy(), want_out)
    assert counts.cpu().tolist() == want_counts.tolist()
    k, v, q, sl = oracle_inputs(inp)
    o_out, _, o_counts, p = orc.decode_attention(6, 4, G, sl, q, orc.quantize_kv(6, 4, G, k, v, sl),
                                                 cfg.softmax_scale, cfg.tau, want_p=True)
    assert_attention_close(out.cpu().numpy(), o_out, vmax(inp), "paged full size vs oracle")
    if not (np.abs(p - np.float32(cfg.tau)) < 1e-7).any():
        assert counts.cpu().tolist() == o_counts.tolist()
