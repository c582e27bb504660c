"""lkv_decode_attention_static -- the decode with its scratch in a fixed
device array inside liblkv instead of a caller workspace -- against
lkv_decode_attention on the same packed cache.  Two calls in a row must
both agree with the workspace entry point within the parity tolerance, and
a failed call must leave nothing behind for the next one.  This file is
collected last so that it also runs after every other test in the process."""
import numpy as np
import pytest
import torch

from gpu_helpers import (assert_attention_close, assert_masks_match, dev, gpu_decode, gpu_quantize, oracle_inputs,
                         vmax)
from quantized_kv_cache_lkv_b200 import lkv
from quantized_kv_cache_lkv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def static_decode(kb, vb, G, inp, cache, softmax_scale, tau, seq_lens=None):
    B, Hq, D = inp["q"].shape
    Hkv, T_cap = cache["k_codes"].shape[1], cache["k_codes"].shape[2]
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    mask = torch.zeros(B, Hq, T_cap, dtype=torch.uint8, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    sl = dev(inp["seq_lens"] if seq_lens is None else seq_lens)
    lkv.lkv_decode_attention_static((kb, vb, G), B, Hq, Hkv, T_cap, D, sl, dev(inp["q"]),
                                    cache["k_codes"], cache["k_sz"], cache["v_codes"], cache["v_sz"],
                                    softmax_scale, tau, out, mask, counts, status)
    torch.cuda.synchronize()
    return out.cpu().numpy(), mask.cpu().numpy(), counts.cpu().numpy(), int(status.item())


@pytest.mark.parametrize("name,cfg,tau", [
    # the Llama-3.1-8B-shaped decode: B16, 32 q / 8 kv heads, D128, T8192
    ("llama8b", W.CONFIGS[2], 1e-4),
    # a ragged batch with groups of 8 query heads (the three-launch path)
    ("ragged_r8", W.Config("ragged_r8", B=3, Hq=16, Hkv=2, D=128, T_cap=700, G=64, bits=[(6, 4)],
                           hh_frac=0.01, seed=91), 1e-3),
])
def test_static_matches_workspace_entry_point_twice(orc, name, cfg, tau):
    inp = W.make_inputs(cfg)
    need = lkv.lkv_decode_workspace_bytes((6, 4, cfg.G), cfg.B, cfg.Hq, cfg.Hkv, cfg.T_cap, cfg.D)
    assert 0 < need <= lkv.LKV_STATIC_WORKSPACE_BYTES
    cache = gpu_quantize(6, 4, cfg.G, inp)
    want_out, want_mask, want_counts = gpu_decode(6, 4, cfg.G, inp, cache, cfg.softmax_scale, tau)
    for call in range(2):
        out, mask, counts, status = static_decode(6, 4, cfg.G, inp, cache, cfg.softmax_scale, tau)
        what = f"{name} call {call}"
        assert status == lkv.LKV_OK, what
        assert_attention_close(out, want_out, vmax(inp), what)
        np.testing.assert_array_equal(mask, want_mask, err_msg=what)
        assert counts.tolist() == want_counts.tolist(), what
    # and against the oracle, which quantizes from bf16 itself: every sequence
    k, v, q, sl = oracle_inputs(inp)
    o_out, o_mask, o_counts, p = orc.decode_attention(6, 4, cfg.G, sl, q, orc.quantize_kv(6, 4, cfg.G, k, v, sl),
                                                      cfg.softmax_scale, tau, want_p=True)
    assert_attention_close(out, o_out, vmax(inp), f"{name} vs oracle")
    if assert_masks_match(mask, o_mask, p, np.float32(tau), sl, f"{name} vs oracle") == 0:
        assert counts.tolist() == o_counts.tolist()


def test_static_failed_call_leaves_nothing_behind(orc):
    """A length beyond T_cap is reported in the status word of that call only;
    the next call on the same scratch is clean and correct."""
    cfg = W.Config("bad", B=2, Hq=8, Hkv=2, D=128, T_cap=512, G=64, bits=[(6, 4)], seed=17)
    inp = W.make_inputs(cfg)
    cache = gpu_quantize(6, 4, 64, inp)
    bad = torch.tensor([512, 513], dtype=torch.int32)
    out, _, _, status = static_decode(6, 4, 64, inp, cache, cfg.softmax_scale, 0.0, seq_lens=bad)
    assert status == lkv.LKV_ERR_INVALID_ARG
    assert np.isfinite(out).all()              # clamped to T_cap, no fault
    want_out, _, want_counts = gpu_decode(6, 4, 64, inp, cache, cfg.softmax_scale, 0.0)
    out, _, counts, status = static_decode(6, 4, 64, inp, cache, cfg.softmax_scale, 0.0)
    assert status == lkv.LKV_OK
    assert_attention_close(out, want_out, vmax(inp), "after a failed call")
    assert counts.tolist() == want_counts.tolist()
    k, v, q, sl = oracle_inputs(inp)
    o_out, _, o_counts = orc.decode_attention(6, 4, 64, sl, q, orc.quantize_kv(6, 4, 64, k, v, sl),
                                              cfg.softmax_scale, 0.0)
    assert_attention_close(out, o_out, vmax(inp), "after a failed call, vs oracle")
    assert counts.tolist() == o_counts.tolist()
