"""The seeded input recipe: the generators draw what the workload description
says they draw (K channel scales log-uniform in [0.5, 4] with two x15
outlier channels per KV head, N(0, 1) V and q, heavy-hitter keys along the
group's mean query, a Zipf(1.1) previous-step mass, ragged lengths in their
ranges), and the same seed gives the same inputs."""
import math

import numpy as np
import pytest
import torch

from quantized_kv_cache_lkv_b200 import workloads as W


def cfg_small(**kw):
    base = dict(name="recipe", B=2, Hq=8, Hkv=2, D=64, T_cap=4096, G=32, bits=[(6, 4)], seed=5)
    base.update(kw)
    return W.Config(**base)


def test_same_seed_same_inputs_other_seed_other_inputs():
    cfg = cfg_small(T_cap=512, hh_frac=0.01)
    a, b = W.make_inputs(cfg, with_mass=True), W.make_inputs(cfg, with_mass=True)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    c = W.make_inputs(W.scaled(cfg, seed=6))
    assert not torch.equal(a["k"], c["k"]) and not torch.equal(a["q"], c["q"])


def test_shapes_dtypes_and_zero_tail():
    cfg = cfg_small(T_cap=300)
    inp = W.make_inputs(cfg, seq_lens=torch.tensor([300, 17], dtype=torch.int32), with_mass=True)
    assert inp["q"].shape == (2, 8, 64) and inp["q"].dtype == torch.bfloat16
    assert inp["k"].shape == inp["v"].shape == (2, 2, 300, 64) and inp["k"].dtype == torch.bfloat16
    assert inp["mass"].shape == (2, 2, 300) and inp["mass"].dtype == torch.float32
    for key in ("k", "v", "mass"):
        assert not inp[key][1, :, 17:].any(), key


def test_k_channel_scales_and_outliers():
    """Per (KV head, channel) the sample std of K is s in [0.5, 4], except
    exactly two channels per head at 15 s in [7.5, 60] (4096 samples each:
    the sample std is within a few percent of s)."""
    inp = W.make_inputs(cfg_small(B=1))
    std = inp["k"][0].float().std(dim=1)  # [Hkv, D]
    for g in range(std.shape[0]):
        out = std[g] > 5.0
        assert int(out.sum()) == 2, g
        assert float(std[g][~out].min()) > 0.5 * 0.93 and float(std[g][~out].max()) < 4.0 * 1.07
        assert float(std[g][out].min()) > 7.5 * 0.93 and float(std[g][out].max()) < 60.0 * 1.07
    # log-uniform: about half of the ordinary channels lie below the geometric mean sqrt(2)
    below = float((std[std < 5.0] < math.sqrt(2.0)).float().mean())
    assert 0.35 < below < 0.65


def test_v_and_q_standard_normal():
    inp = W.make_inputs(cfg_small(B=1))
    for key in ("v", "q"):
        x = inp[key].float().flatten()
        assert abs(float(x.mean())) < 0.05 * (1 if key == "v" else 3), key
        assert abs(float(x.std()) - 1.0) < 0.03 * (1 if key == "v" else 3), key


def test_heavy_hitters_follow_the_group_mean_query():
    """round(f T) positions per sequence, the same for every KV head, whose K
    row is 4 * mean(q of the group) + N(0, 1); no other row is near it."""
    cfg = cfg_small(B=2, D=128, hh_frac=0.01)  # 128 channels: a hitter's residual RMS is 1 +- 0.06
    inp = W.make_inputs(cfg)
    r = cfg.Hq // cfg.Hkv
    for b in range(cfg.B):
        qbar = inp["q"][b].float().view(cfg.Hkv, r, cfg.D).mean(dim=1)
        sets = []
        for g in range(cfg.Hkv):
            res = (inp["k"][b, g].float() - 4.0 * qbar[g]).pow(2).mean(dim=1).sqrt()  # [T]
            hh = torch.nonzero(res < 1.7).flatten()  # hitters near 1, other rows above 2
            assert len(hh) == round(0.01 * cfg.T_cap), (b, g)
            assert float(res[hh].mean()) == pytest.approx(1.0, abs=0.1)
            sets.append(set(hh.tolist()))
        assert all(s == sets[0] for s in sets), b


def test_mass_is_a_zipf_law_over_a_permutation():
    """Per (sequence, KV head) the mass sums to 1 over T_b and, sorted, is
    r^-1.1 / sum r^-1.1 for r = 1..T_b."""
    cfg = cfg_small(T_cap=1000)
    lens = torch.tensor([1000, 333], dtype=torch.int32)
    mass = W.make_inputs(cfg, seq_lens=lens, with_mass=True)["mass"]
    for b in range(cfg.B):
        T = int(lens[b])
        ranks = np.arange(1, T + 1, dtype=np.float64)
        want = (ranks ** -1.1 / (ranks ** -1.1).sum()).astype(np.float32)
        for g in range(cfg.Hkv):
            m = mass[b, g, :T].numpy()
            np.testing.assert_array_equal(np.sort(m)[::-1], want)
            assert abs(float(m.astype(np.float64).sum()) - 1.0) < 1e-5
        assert not torch.equal(mass[b, 0, :T], mass[b, 1, :T])  # each head its own ranking


def test_ragged_lengths_stay_in_their_ranges():
    for cid in (4, 5):
        base = W.CONFIGS[cid]
        cfg = W.scaled(base, B=400, T_cap=base.seq_hi)
        lens = W.seq_lens_for(cfg, torch.Generator().manual_seed(cfg.seed)).numpy()
        assert lens.min() >= base.seq_lo and lens.max() <= base.seq_hi
        if base.seq == "uniform":
            mid = (base.seq_lo + base.seq_hi) / 2
        else:  # log-uniform: the geometric midpoint splits the lengths in half
            mid = math.sqrt(base.seq_lo * base.seq_hi)
        assert 0.4 < float((lens < mid).mean()) < 0.6, cid
