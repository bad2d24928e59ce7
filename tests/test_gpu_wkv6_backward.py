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


@pytest.mark.parametrize("finch", [False, True])
@pytest.mark.parametrize("which", ["s_in", "gs_out"])
def test_backward_one_state_only(cuda_device, finch, which):
    # an initial state without a final-state gradient, and the reverse (the Eagle backward too)
    B, T, H = 2, 90, 2
    p = (wi.wkv6_problem if finch else wi.wkv5_problem)(B, T, H, 64, seed=102)
    g = wi.wkv5_grads(B, T, H, 64, seed=103, states=True)
    g.pop("gs_out" if which == "s_in" else "s_in")
    c = {k: v.to(cuda_device) for k, v in list(p.items()) + list(g.items())}
    bwd = rw.rwkv_wkv6_backward if finch else rw.rwkv_wkv5_backward
    out = bwd(c["r"], c["k"], c["v"], c["omega"], c["u"], c["gy"], c.get("s_in"), c.get("gs_out"), want_gs_in=True)
    rw.rwkv_check_device_error()
    ref = (oracle.wkv6_backward if finch else oracle.wkv5_backward)(
        p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], s_in=g.get("s_in"), gs_out=g.get("gs_out"))
    if finch:
        _check(out, ref, which + " only: ")
    else:
        for got, want, name in zip(out, ref, ("gr", "gk", "gv", "gomega", "gu", "gs_in")):
            assert_close_rms(got.cpu(), want, TOL_BF16, f"{which} only: {name}")


@pytest.mark.parametrize("finch", [False, True])
def test_backward_resumes_across_a_split(cuda_device, finch):
    # the backward of a sequence is the backward of its two halves chained through the state: the
    # first half's final state is the second half's s_in, and the second half's gs_in is the first
    # half's gs_out.  Per-token gradients then agree with the whole-sequence call, and the batch and
    # time sums (gu; Eagle's gomega) are the sums of the halves'
    B, T, H, T1 = 2, 200, 2, 77
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    p = {k: v.to(cuda_device) for k, v in gen(B, T, H, 64, seed=104).items()}
    g = {k: v.to(cuda_device) for k, v in wi.wkv5_grads(B, T, H, 64, seed=105, states=True).items()}
    fwd = rw.rwkv_wkv6_forward if finch else rw.rwkv_wkv5_forward
    bwd = rw.rwkv_wkv6_backward if finch else rw.rwkv_wkv5_backward

    def part(x, a, b):  # tokens [a, b) of a [B,T,H,N] tensor (omega too for Finch)
        return x[:, a:b].contiguous()

    om = (lambda a, b: part(p["omega"], a, b)) if finch else (lambda a, b: p["omega"])
    whole = bwd(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g["s_in"], g["gs_out"], want_gs_in=True)
    _, s_mid = fwd(part(p["r"], 0, T1), part(p["k"], 0, T1), part(p["v"], 0, T1), om(0, T1), p["u"], g["s_in"],
                   return_state=True)
    second = bwd(part(p["r"], T1, T), part(p["k"], T1, T), part(p["v"], T1, T), om(T1, T), p["u"],
                 part(g["gy"], T1, T), s_mid, g["gs_out"], want_gs_in=True)
    first = bwd(part(p["r"], 0, T1), part(p["k"], 0, T1), part(p["v"], 0, T1), om(0, T1), p["u"],
                part(g["gy"], 0, T1), g["s_in"], second[5], want_gs_in=True)
    rw.rwkv_check_device_error()
    names = ("gr", "gk", "gv")
    for i, name in enumerate(names):
        joined = torch.cat([first[i], second[i]], dim=1)
        assert_close_rms(joined.cpu(), whole[i].cpu().double().numpy(), 2 * TOL_BF16, name)
    if finch:
        joined = torch.cat([first[3], second[3]], dim=1)
        assert_close_rms(joined.cpu(), whole[3].cpu().double().numpy(), 2 * TOL_BF16, "gomega")
    else:
        assert_close_rms((first[3] + second[3]).cpu(), whole[3].cpu().double().numpy(), 2 * TOL_BF16, "gomega")
    assert_close_rms((first[4] + second[4]).cpu(), whole[4].cpu().double().numpy(), 2 * TOL_BF16, "gu")
    assert_close_rms(first[5].cpu(), whole[5].cpu().double().numpy(), 2 * TOL_BF16, "gs_in")
