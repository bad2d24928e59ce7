"""Edge cases of the CUDA path on a B200: non-finite inputs stay where the
formulas put them (values are data, nothing is validated or clamped), and
problems past 2^31 elements, whose last outputs sit at 64-bit offsets, match
the oracle there."""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import TOL_BF16, TOL_GRAD, TOL_Y, assert_close_abs1, assert_close_rms, state_to_ab

pytestmark = pytest.mark.gpu


def _cuda(p, dev):
    return {k: v.to(dev) for k, v in p.items()}


@pytest.mark.parametrize("algo", [rw.ALGO_SEQUENTIAL, rw.ALGO_CHUNKED])
def test_wkv4_nan_key_stays_in_its_lane(cuda_device, algo):
    # a NaN key at (b=1, t=100, c=5): that lane's outputs from t = 100 on are NaN (the key enters the
    # state); every other lane, and the lane's outputs before the 16-step segment of t = 100, are exactly
    # those of the clean run; t = 96..99 may round differently (the segment's power-of-two scale is
    # taken over its finite keys) and stay within the fp32 tolerance
    B, T, C = 2, 300, 64
    p = _cuda(wi.wkv4_problem(B, T, C, 51), cuda_device)
    y0 = rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"], p["v"], algo=algo)
    k = p["k"].clone()
    k[1, 100, 5] = float("nan")
    y1 = rw.rwkv_wkv4_forward(p["w"], p["u"], k, p["v"], algo=algo)
    assert torch.isnan(y1[1, 100:, 5]).all()
    assert torch.equal(y1[1, :96, 5], y0[1, :96, 5])
    assert_close_abs1(y1[1, 96:100, 5], y0[1, 96:100, 5].double().cpu().numpy(), TOL_Y, "t = 96..99")
    mask = torch.ones_like(y1, dtype=torch.bool)
    mask[1, :, 5] = False
    assert torch.equal(y1[mask], y0[mask])


def test_wkv4_step_nan_key_stays_in_its_lane(cuda_device):
    # one decode step with a NaN key in lane (2, 9): that lane's output and state turn NaN, every other
    # lane's output and state are exactly those of the clean step
    B, C = 4, 128
    p = _cuda(wi.wkv4_problem(B, 3, C, 56), cuda_device)
    _, st = rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"][:, :2].contiguous(), p["v"][:, :2].contiguous(),
                                 return_state=True)
    k1, v1 = p["k"][:, 2].contiguous(), p["v"][:, 2].contiguous()
    s0 = st.clone()
    y0 = rw.rwkv_wkv4_step(p["w"], p["u"], k1, v1, s0)
    kn = k1.clone()
    kn[2, 9] = float("nan")
    s1 = st.clone()
    y1 = rw.rwkv_wkv4_step(p["w"], p["u"], kn, v1, s1)
    assert torch.isnan(y1[2, 9]) and torch.isnan(s1[0, 2, 9]) and torch.isnan(s1[1, 2, 9])
    mask = torch.ones_like(y1, dtype=torch.bool)
    mask[2, 9] = False
    assert torch.equal(y1[mask], y0[mask])
    assert torch.equal(s1[:, mask], s0[:, mask])


def test_wkv5_nan_receptance_stays_in_its_token(cuda_device):
    # r only reads the state: a NaN in r at (b=0, t=70, h=1) makes exactly that token's output row NaN
    B, T, H = 2, 200, 3
    p = _cuda(wi.wkv5_problem(B, T, H, 64, seed=52), cuda_device)
    y0, s0 = rw.rwkv_wkv5_forward(**p, return_state=True)
    r = p["r"].clone()
    r[0, 70, 1, 3] = float("nan")
    y1, s1 = rw.rwkv_wkv5_forward(r, p["k"], p["v"], p["omega"], p["u"], return_state=True)
    assert torch.isnan(y1[0, 70, 1].float()).all()
    mask = torch.ones_like(y1, dtype=torch.bool)
    mask[0, 70, 1] = False
    assert torch.equal(y1[mask], y0[mask])
    assert torch.equal(s1, s0)


def test_wkv6_nan_decay_enters_the_state(cuda_device):
    # a NaN omega at (b=1, t=90, h=0, n=7) decays row 7 of that head's state by NaN from token 90 on:
    # the head's outputs after token 90 are NaN.  The chunk holding it (tokens 64..127) fails the range
    # check and runs the per-token recurrence, so tokens 64..90 match the clean run within the bf16
    # tolerance; earlier chunks and every other head are unchanged bit for bit
    B, T, H = 2, 200, 2
    p = _cuda(wi.wkv6_problem(B, T, H, 64, seed=53), cuda_device)
    y0 = rw.rwkv_wkv6_forward(**p)
    om = p["omega"].clone()
    om[1, 90, 0, 7] = float("nan")
    y1 = rw.rwkv_wkv6_forward(p["r"], p["k"], p["v"], om, p["u"])
    assert torch.isnan(y1[1, 91:, 0].float()).all()
    assert torch.equal(y1[1, :64, 0], y0[1, :64, 0])
    assert_close_rms(y1[1, 64:91, 0], y0[1, 64:91, 0].float().cpu().double().numpy(), TOL_BF16, "t = 64..90")
    mask = torch.ones_like(y1, dtype=torch.bool)
    mask[1, :, 0] = False
    assert torch.equal(y1[mask], y0[mask])


@pytest.mark.parametrize("finch", [False, True])
def test_matrix_state_backward_nan_stays_in_its_head(cuda_device, finch):
    # a NaN in gy at (b=1, t=120, h=2, j=5): every gradient of that (batch row, head) may turn NaN,
    # and gomega / gu of head 2 (sums over the batch); every other (batch row, head) and the other
    # heads' sums are bit for bit those of the clean run
    B, T, H = 2, 200, 3
    p = _cuda((wi.wkv6_problem if finch else wi.wkv5_problem)(B, T, H, 64, seed=54), cuda_device)
    g = _cuda(wi.wkv5_grads(B, T, H, 64, seed=55, states=True), cuda_device)
    bwd = rw.rwkv_wkv6_backward if finch else rw.rwkv_wkv5_backward
    clean = bwd(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g["s_in"], g["gs_out"], want_gs_in=True)
    gy = g["gy"].clone()
    gy[1, 120, 2, 5] = float("nan")
    dirty = bwd(p["r"], p["k"], p["v"], p["omega"], p["u"], gy, g["s_in"], g["gs_out"], want_gs_in=True)
    rw.rwkv_check_device_error()
    assert torch.isnan(dirty[0][1, 120, 2].float()).any()  # gr of the token itself
    for i, name in enumerate(("gr", "gk", "gv")):
        m = torch.ones_like(dirty[i], dtype=torch.bool)
        m[1, :, 2] = False
        assert torch.equal(dirty[i][m], clean[i][m]), name
    om_clean, om_dirty = clean[3], dirty[3]
    if finch:  # per token: the other (batch row, head) pairs
        m = torch.ones_like(om_dirty, dtype=torch.bool)
        m[1, :, 2] = False
        assert torch.equal(om_dirty[m], om_clean[m]), "gomega"
    else:  # per head, summed over the batch
        assert torch.equal(om_dirty[:2], om_clean[:2]), "gomega"
    assert torch.equal(dirty[4][:2], clean[4][:2]), "gu"
    m = torch.ones_like(dirty[5], dtype=torch.bool)
    m[1, 2] = False
    assert torch.equal(dirty[5][m], clean[5][m]), "gs_in"


def test_wkv4_past_2pow31_elements(cuda_device):
    # B=2, T=2^19+2^12, C=2048 fp32: 2.16e9 elements per tensor.  The last 2048 steps of batch 1 (the
    # highest offsets) against the oracle from the GPU's own state before them, for 8 channels;
    # gk, gv of those steps likewise (they depend only on the state there and later inputs).
    B, T, C, W = 2, (1 << 19) + (1 << 12), 2048, 2048
    assert B * T * C > 2 ** 31
    p = wi.wkv4_problem(B, T, C, 54, with_gy=True, device=cuda_device)
    y, ck = rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"], p["v"], checkpoints=True)
    gk, gv, _, _ = rw.rwkv_wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["gy"], ckpt=ck)
    rw.rwkv_check_device_error()
    chans = torch.arange(3, C, C // 8)[:8]
    win = {n: p[n][1:2, T - W:, :][:, :, chans.to(cuda_device)].cpu() for n in ("k", "v", "gy")}
    y_win = y[1:2, T - W:, :][:, :, chans.to(cuda_device)].cpu()
    gk_win = gk[1:2, T - W:, :][:, :, chans.to(cuda_device)].cpu()
    gv_win = gv[1:2, T - W:, :][:, :, chans.to(cuda_device)].cpu()
    del y, gk, gv, ck
    # the state before the window, from the forward over batch 1's prefix
    _, st = rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"][1:2, :T - W].contiguous(),
                                 p["v"][1:2, :T - W].contiguous(), return_state=True)
    ab = state_to_ab(st)[:, :, chans.to(cuda_device)].cpu().numpy()
    w, u = p["w"][chans.to(cuda_device)].cpu(), p["u"][chans.to(cuda_device)].cpu()
    ref_y = oracle.wkv4_forward(w, u, win["k"], win["v"], state_in=ab)
    assert_close_abs1(y_win, ref_y, TOL_Y, "y at 64-bit offsets")
    ref_g = oracle.wkv4_backward(w, u, win["k"], win["v"], win["gy"], state_in=ab)
    assert_close_abs1(gk_win, ref_g[0], TOL_GRAD, "gk at 64-bit offsets")
    assert_close_abs1(gv_win, ref_g[1], TOL_GRAD, "gv at 64-bit offsets")


@pytest.mark.parametrize("finch", [False, True])
def test_matrix_state_past_2pow31_elements(cuda_device, finch):
    # B=2, T=2^20+2^12, H=16, N=64: 2.16e9 elements per tensor.  The last 256 tokens of (b=1, h=15)
    # against the oracle from the GPU's own state before them.
    B, T, H, N, W = 2, (1 << 20) + (1 << 12), 16, 64, 256
    assert B * T * H * N > 2 ** 31
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    fwd = rw.rwkv_wkv6_forward if finch else rw.rwkv_wkv5_forward
    p = gen(B, T, H, N, seed=55, device=cuda_device)
    y = fwd(**p)
    rw.rwkv_check_device_error()
    y_win = y[1:2, T - W:, 15:16].cpu()
    del y
    pre = {n: p[n][1:2, :T - W].contiguous() for n in ("r", "k", "v")}
    om_pre = p["omega"][1:2, :T - W].contiguous() if finch else p["omega"]
    _, s = fwd(pre["r"], pre["k"], pre["v"], om_pre, p["u"], return_state=True)
    del pre
    s15 = s[:, 15:16].cpu().double().numpy()
    win = {n: p[n][1:2, T - W:, 15:16].cpu() for n in ("r", "k", "v")}
    if finch:
        ref = oracle.wkv6_forward(win["r"], win["k"], win["v"], p["omega"][1:2, T - W:, 15:16].cpu(),
                                  p["u"][15:16].cpu(), s_in=s15)
    else:
        ref = oracle.wkv5_forward(win["r"], win["k"], win["v"], p["omega"][15:16].cpu(), p["u"][15:16].cpu(),
                                  s_in=s15)
    assert_close_rms(y_win, ref, TOL_BF16, "y at 64-bit offsets")
