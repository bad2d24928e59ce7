"""GPU parity of the Finch / RWKV-6 backward (rwkv_wkv6_backward) against the fp64
oracle's backward, through the C-ABI.  gr, gk, gv are bf16 and gomega (one value per
token and channel), gu, gs_in fp32; every one is held to the bf16 rule of the forward
tests, |got - ref| <= 8e-3 * max(|ref|, rms(ref)), per head for the per-head tensors."""
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import TOL_BF16, assert_close_rms

pytestmark = pytest.mark.gpu
SEED = wi.CONFIG_SEED_BASE


def _run(p, g, dev):
    c = {k: v.to(dev) for k, v in p.items()}
    gg = {k: v.to(dev) for k, v in g.items()}
    out = rw.rwkv_wkv6_backward(c["r"], c["k"], c["v"], c["omega"], c["u"], gg["gy"], gg.get("s_in"),
                                gg.get("gs_out"), want_gs_in=True)
    rw.rwkv_check_device_error()
    ref = oracle.wkv6_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], s_in=g.get("s_in"),
                               gs_out=g.get("gs_out"))
    return out, ref


def _check(out, ref, what=""):
    gr, gk, gv, gom, gu, gsi = (x.cpu() for x in out)
    rr, rk, rv, rom, ru, rsi = ref
    B, T, H, N = gr.shape
    for b in range(B):
        for h in range(H):
            for got, want, name in ((gr, rr, "gr"), (gk, rk, "gk"), (gv, rv, "gv"), (gom, rom, "gomega")):
                assert_close_rms(got[b, :, h], want[b, :, h], TOL_BF16, f"{what}{name} head ({b},{h})")
            assert_close_rms(gsi[b, h], rsi[b, h], TOL_BF16, f"{what}gs_in head ({b},{h})")
    assert_close_rms(gu, ru, TOL_BF16, what + "gu")


@pytest.mark.parametrize("states", [False, True])
@pytest.mark.parametrize("shape", [(1, 64, 1), (1, 100, 2), (2, 33, 3), (1, 1, 1), (2, 200, 3), (1, 128, 2),
                                   (1, 72, 1), (1, 9, 2)])
def test_backward_small(cuda_device, shape, states):
    # whole, ragged and single chunks; sub-chunks of 8 tokens cut at every remainder
    B, T, H = shape
    p = wi.wkv6_problem(B, T, H, 64, seed=90)
    g = wi.wkv5_grads(B, T, H, 64, seed=91, states=states)
    out, ref = _run(p, g, cuda_device)
    _check(out, ref)


@pytest.mark.parametrize("omega_range", [(-8.0, -4.0), (-3.0, 0.69), (-1.0, 2.0), (2.0, 3.0)])
def test_backward_decay_ranges(cuda_device, omega_range):
    # slow to fast per-token decays (w down to e^-20 and below with the jitter)
    p = wi.wkv6_problem(2, 150, 3, 64, seed=92, omega_range=omega_range)
    g = wi.wkv5_grads(2, 150, 3, 64, seed=93, states=True)
    out, ref = _run(p, g, cuda_device)
    _check(out, ref, f"omega {omega_range}: ")


def test_backward_zero_decay_tokens(cuda_device):
    # tokens with w = 0 exactly (omega = 100: exp(-exp(100)) underflows) cut the state; their
    # gomega is 0 (dw/domega = -e^omega w = 0 in the oracle too)
    B, T, H = 1, 130, 2
    p = wi.wkv6_problem(B, T, H, 64, seed=94)
    om = p["omega"].clone()
    om[:, 7::23] = 100.0
    p["omega"] = om
    g = wi.wkv5_grads(B, T, H, 64, seed=95, states=True)
    out, ref = _run(p, g, cuda_device)
    _check(out, ref)


def test_backward_constant_decay_is_eagle(cuda_device):
    # with the same omega at every token the Finch backward is the Eagle backward (its per-token
    # gomega summed over batch and time gives Eagle's gomega)
    B, T, H = 2, 140, 2
    p = wi.wkv5_problem(B, T, H, 64, seed=96)
    g = wi.wkv5_grads(B, T, H, 64, seed=97, states=True)
    c = {k: v.to(cuda_device) for k, v in p.items()}
    gg = {k: v.to(cuda_device) for k, v in g.items()}
    om_t = c["omega"].expand(B, T, H, 64).contiguous()
    f = rw.rwkv_wkv6_backward(c["r"], c["k"], c["v"], om_t, c["u"], gg["gy"], gg["s_in"], gg["gs_out"],
                              want_gs_in=True)
    e = rw.rwkv_wkv5_backward(c["r"], c["k"], c["v"], c["omega"], c["u"], gg["gy"], gg["s_in"], gg["gs_out"],
                              want_gs_in=True)
    for i, name in enumerate(("gr", "gk", "gv")):
        assert_close_rms(f[i].cpu(), e[i].cpu(), 2 * TOL_BF16, name)
    assert_close_rms(f[3].sum(dim=(0, 1)).cpu(), e[3].cpu(), 2 * TOL_BF16, "gomega summed")
    assert_close_rms(f[4].cpu(), e[4].cpu(), 2 * TOL_BF16, "gu")
    assert_close_rms(f[5].cpu(), e[5].cpu(), 2 * TOL_BF16, "gs_in")


def test_backward_empty_and_no_gs_in(cuda_device):
    p = {k: v.to(cuda_device) for k, v in wi.wkv6_problem(2, 0, 3, 64, seed=98).items()}
    g = wi.wkv5_grads(2, 0, 3, 64, seed=99, states=True, device=cuda_device)
    gr, gk, gv, gom, gu, gsi = rw.rwkv_wkv6_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"],
                                                     g["s_in"], g["gs_out"], want_gs_in=True)
    assert gr.numel() == 0 and gom.numel() == 0
    assert torch.equal(gu, torch.zeros_like(gu))
    assert torch.equal(gsi, g["gs_out"])
    p = {k: v.to(cuda_device) for k, v in wi.wkv6_problem(1, 50, 2, 64, seed=98).items()}
    g = wi.wkv5_grads(1, 50, 2, 64, seed=99, device=cuda_device)
    a = rw.rwkv_wkv6_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"])
    b = rw.rwkv_wkv6_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], want_gs_in=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_deterministic(cuda_device):
    p = {k: v.to(cuda_device) for k, v in wi.wkv6_problem(2, 300, 3, 64, seed=100).items()}
    g = wi.wkv5_grads(2, 300, 3, 64, seed=101, states=True, device=cuda_device)
    a = rw.rwkv_wkv6_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g["s_in"], g["gs_out"])
    b = rw.rwkv_wkv6_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g["s_in"], g["gs_out"])
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_workload_full_size(cuda_device):
    # B4 T4096 H40 N64 (the Finch forward workload) with gy ~ N(0, 1): every head of gr, gk, gv and
    # gomega and every channel of gu against the oracle
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv6_problem(B, T, H, N, seed=SEED + 6)
    g = wi.wkv5_grads(B, T, H, N, seed=SEED + 10)
    out, ref = _run(p, g, cuda_device)
    _check(out, ref)


def test_backward_fast_decay_full_size(cuda_device):
    # the same workload with the channel base omega ~ U(-1, 2): many tokens decay faster than any
    # chunked factorization could take
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv6_problem(B, T, H, N, seed=SEED + 7, omega_range=(-1.0, 2.0))
    g = wi.wkv5_grads(B, T, H, N, seed=SEED + 11, states=True)
    out, ref = _run(p, g, cuda_device)
    _check(out, ref)
