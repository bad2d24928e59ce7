"""The seeded input generator: published SplitMix64 outputs, sub-block
regeneration and the configured distributions."""
import math

import torch

import wkv_inputs as wi


def test_splitmix64_published_sequence():
    # SplitMix64 reference implementation seeded with 1234567: its first five
    # outputs are mix(seed + i * 0x9E3779B97F4A7C15), i = 1..5.
    expect = [6457827717110365317, 3203168211198807973, 9817491932198370423,
              4593380528125082431, 16408922859458223821]
    got = wi._mix(wi._s64(1234567) + (torch.arange(5) + 1) * wi._s64(wi._GAMMA))
    assert [x & ((1 << 64) - 1) for x in got.tolist()] == expect
    assert [wi.splitmix64_scalar(1234567 + i * wi._GAMMA) for i in range(1, 6)] == expect


def test_subblock_regenerates_same_values():
    B, T, C, seed = 3, 50, 40, 99
    full = wi.btc_field("k", seed, B, T, C, outliers=True)
    part = wi.btc_field("k", seed, B, T, C, t0=17, t1=29, outliers=True)
    assert torch.equal(full[:, 17:29], part)
    b_sel, c_sel = torch.tensor([0, 2, 1]), torch.tensor([5, 39, 0])
    lanes = wi.btc_field("k", seed, B, T, C, b_sel=b_sel, c_sel=c_sel, outliers=True)
    assert torch.equal(lanes, full[b_sel, :, c_sel].T)


def test_distributions():
    n = 1 << 20
    idx = torch.arange(n)
    x = wi.normal(5, 3, idx)
    assert abs(x.mean().item()) < 5e-3 and abs(x.std().item() - 1) < 5e-3
    u = wi.uniform(5, 3, idx)
    assert 0.0 <= u.min().item() and u.max().item() < 1.0
    k = wi.btc_field("k", 7, 4, 256, 1024, outliers=True)
    frac = (k.abs() >= 20).double().mean().item()
    assert abs(frac - 0.01) < 1e-3 and k.abs().max().item() <= 40.0
    w, uu = wi.wkv4_params(7, 4096)
    assert 0.01 <= w.min().item() and w.max().item() <= 5.0
    # log-uniform: the median of log w sits at the midpoint of [ln .01, ln 5]
    mid = 0.5 * (math.log(0.01) + math.log(5.0))
    assert abs(torch.log(w.double()).median().item() - mid) < 0.1
    assert -1.0 <= uu.min().item() and uu.max().item() <= 1.0
    p = wi.wkv5_problem(1, 8, 2, 64, seed=3)
    assert p["r"].dtype == torch.bfloat16 and p["r"].shape == (1, 8, 2, 64)
    assert -6.0 <= p["omega"].min().item() and p["omega"].max().item() <= 0.0
