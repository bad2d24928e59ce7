"""GPU parity of the Eagle / RWKV-5 backward (rwkv_wkv5_backward) against the fp64
oracle's backward, through the C-ABI.  gr, gk, gv are bf16 and gomega, gu, gs_in
fp32; every one is held to the bf16 rule of the forward tests,
|got - ref| <= 8e-3 * max(|ref|, rms(ref)), per head for the per-head tensors."""
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import TOL_BF16, assert_close_rms

pytestmark = pytest.mark.gpu
SEED = wi.CONFIG_SEED_BASE


def _run(p, g, dev, states):
    c = {k: v.to(dev) for k, v in p.items()}
    gg = {k: v.to(dev) for k, v in g.items()}
    out = rw.rwkv_wkv5_backward(c["r"], c["k"], c["v"], c["omega"], c["u"], gg["gy"], gg.get("s_in"),
                                gg.get("gs_out"), want_gs_in=True)
    rw.rwkv_check_device_error()
    ref = oracle.wkv5_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], s_in=g.get("s_in"),
                               gs_out=g.get("gs_out"))
    return out, ref


def _check(out, ref, what=""):
    names = ("gr", "gk", "gv", "gomega", "gu", "gs_in")
    gr, gk, gv, gom, gu, gsi = (x.cpu() for x in out)
    rr, rk, rv, rom, ru, rsi = ref
    B, T, H, N = gr.shape
    for b in range(B):
        for h in range(H):
            for got, want, name in ((gr, rr, "gr"), (gk, rk, "gk"), (gv, rv, "gv")):
                assert_close_rms(got[b, :, h], want[b, :, h], TOL_BF16, f"{what}{name} head ({b},{h})")
            assert_close_rms(gsi[b, h], rsi[b, h], TOL_BF16, f"{what}gs_in head ({b},{h})")
    assert_close_rms(gom, rom, TOL_BF16, what + "gomega")
    assert_close_rms(gu, ru, TOL_BF16, what + "gu")


@pytest.mark.parametrize("states", [False, True])
@pytest.mark.parametrize("shape", [(1, 64, 1), (1, 100, 2), (2, 33, 3), (1, 1, 1), (2, 200, 3), (1, 128, 2)])
def test_backward_small(cuda_device, shape, states):
    B, T, H = shape
    p = wi.wkv5_problem(B, T, H, 64, seed=80)
    g = wi.wkv5_grads(B, T, H, 64, seed=81, states=states)
    out, ref = _run(p, g, cuda_device, states)
    _check(out, ref)


@pytest.mark.parametrize("omega_range", [(-8.0, -4.0), (-3.0, 0.69), (0.3, 0.69), (-1.0, 2.0), (0.7, 2.0), (2.0, 3.0)])
def test_backward_decay_ranges(cuda_device, omega_range):
    # slow, mixed and fast decays: exp(omega) up to 1.99 inside the chunked factorization's range;
    # (-1, 2) mixes in rows above it, (0.7, 2) and (2, 3) (w down to e^-20) have every row above it
    p = wi.wkv5_problem(2, 150, 3, 64, seed=82, omega_range=omega_range)
    g = wi.wkv5_grads(2, 150, 3, 64, seed=83, states=True)
    out, ref = _run(p, g, cuda_device, True)
    _check(out, ref, f"omega {omega_range}: ")


@pytest.mark.parametrize("shape", [(1, 64, 2), (1, 65, 2), (2, 127, 2), (1, 1, 1)])
def test_backward_fast_decay_ragged(cuda_device, shape):
    # fast rows at ragged lengths: the reversed pass's first chunk has `lead` empty positions
    B, T, H = shape
    p = wi.wkv5_problem(B, T, H, 64, seed=84, omega_range=(-1.0, 2.0))
    g = wi.wkv5_grads(B, T, H, 64, seed=85, states=True)
    out, ref = _run(p, g, cuda_device, True)
    _check(out, ref, f"shape {shape}: ")


def test_backward_deterministic(cuda_device):
    p = {k: v.to(cuda_device) for k, v in wi.wkv5_problem(2, 300, 3, 64, seed=86).items()}
    g = wi.wkv5_grads(2, 300, 3, 64, seed=87, states=True, device=cuda_device)
    a = rw.rwkv_wkv5_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g["s_in"], g["gs_out"])
    b = rw.rwkv_wkv5_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g["s_in"], g["gs_out"])
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_workload_full_size(cuda_device):
    # B4 T4096 H40 N64 (the Eagle forward workload) with gy ~ N(0, 1): every head of gr, gk, gv
    # and every channel of gomega, gu against the oracle
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv5_problem(B, T, H, N, seed=SEED + 4)
    g = wi.wkv5_grads(B, T, H, N, seed=SEED + 8)
    out, ref = _run(p, g, cuda_device, False)
    _check(out, ref)


def test_backward_fast_decay_full_size(cuda_device):
    # the same workload with omega ~ U(-1, 2): every head has rows above the factorization's range
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv5_problem(B, T, H, N, seed=SEED + 5, omega_range=(-1.0, 2.0))
    g = wi.wkv5_grads(B, T, H, N, seed=SEED + 9)
    out, ref = _run(p, g, cuda_device, False)
    _check(out, ref)
