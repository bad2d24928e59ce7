"""GPU parity of the receptance-gated WKV-4 forward (o = sigmoid(r) * WKV) and its
backward against the fp64 oracle, through the C-ABI.  Tolerances as the plain
operator: fp32 outputs 1e-5 * max(1, |ref|); gk, gv, gr 1e-4 * max(1, |ref|)
per element; gw, gu per element too; bf16 I/O 8e-3 * max(|ref|, rms(ref))."""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import (TOL_BF16, TOL_Y, assert_close_abs1, assert_close_rms, assert_grads_close, assert_state_close,
                     state_to_ab)

pytestmark = pytest.mark.gpu
SEED = wi.CONFIG_SEED_BASE
ALGOS = [rw.ALGO_SEQUENTIAL, rw.ALGO_CHUNKED]


def _cuda(p, dev):
    return {k: v.to(dev) for k, v in p.items()}


def _check_grads(got, ref, what=""):
    assert_grads_close(got, ref, what, names=("gk", "gv", "gr", "gw", "gu"))


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("shape", [(1, 64, 128), (3, 333, 100), (1, 1, 32), (2, 7, 4), (5, 250, 36)])
def test_gated_forward(cuda_device, algo, shape):
    B, T, C = shape
    p = wi.wkv4_problem(B, T, C, 31, outliers=True, gated=True)
    g = _cuda(p, cuda_device)
    o, st = rw.rwkv_wkv4_forward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], algo=algo, return_state=True)
    assert_close_abs1(o, oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], p["r"]), TOL_Y, "o")
    # the gate does not enter the recurrence: the state is the plain forward's, bitwise on the same
    # schedule.  The chunked schedule of the plain forward runs in one launch (fp64 segment summaries)
    # where the gated one, with three input boxes per stage, keeps three launches (fp32 summaries):
    # there the two agree within the state tolerance.
    _, st0 = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], algo=algo, return_state=True)
    if algo == rw.ALGO_SEQUENTIAL:
        assert torch.equal(st, st0)
    else:
        assert_state_close(st, state_to_ab(st0), "state")


@pytest.mark.parametrize("shape", [(1, 64, 128), (3, 333, 100), (2, 7, 4), (5, 250, 36)])
@pytest.mark.parametrize("use_ckpt", [True, False])
def test_gated_backward(cuda_device, shape, use_ckpt):
    B, T, C = shape
    p = wi.wkv4_problem(B, T, C, 32, outliers=True, with_gy=True, gated=True)
    g = _cuda(p, cuda_device)
    ck = None
    if use_ckpt:
        _, ck = rw.rwkv_wkv4_forward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], checkpoints=True)
    got = rw.rwkv_wkv4_backward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], g["go"], ckpt=ck)
    ref = oracle.wkv4_gated_backward(p["w"], p["u"], p["k"], p["v"], p["r"], p["go"])
    _check_grads(got, ref)


def test_gated_backward_with_initial_state(cuda_device):
    # an initial state (A, B, 0) rounded to fp32, the same values on both sides; checkpoints
    # from the gated forward and recomputed from the state alike
    B, T, C = 2, 90, 64
    p = wi.wkv4_problem(B, T + 30, C, 33, outliers=True, with_gy=True, gated=True)
    _, s0 = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :30], p["v"][:, :30], return_state=True)
    st = torch.zeros(3, B, C)
    st[0], st[1] = torch.from_numpy(s0[0]).float(), torch.from_numpy(s0[1]).float()
    q = {k: (v[:, 30:].contiguous() if v.dim() == 3 else v) for k, v in p.items()}
    g = _cuda(q, cuda_device)
    stg = st.to(cuda_device)
    o, ck = rw.rwkv_wkv4_forward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], stg, checkpoints=True)
    s64 = st.double().numpy()[:2]
    assert_close_abs1(o, oracle.wkv4_gated_forward(q["w"], q["u"], q["k"], q["v"], q["r"], state_in=s64), TOL_Y,
                      "o")
    ref = oracle.wkv4_gated_backward(q["w"], q["u"], q["k"], q["v"], q["r"], q["go"], state_in=s64)
    _check_grads(rw.rwkv_wkv4_backward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], g["go"], ckpt=ck), ref,
                 "ckpt ")
    _check_grads(rw.rwkv_wkv4_backward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], g["go"], state_in=stg), ref,
                 "recompute ")


def test_open_gate_equals_plain_backward_bitwise(cuda_device):
    # sigmoid(40) rounds to 1 in fp32, so gy = go exactly: gk, gv, gw, gu equal the plain backward's bits
    B, T, C = 2, 200, 96
    p = wi.wkv4_problem(B, T, C, 35, outliers=True, with_gy=True, gated=True)
    g = _cuda(p, cuda_device)
    r_open = torch.full_like(g["k"], 40.0)
    o, ck = rw.rwkv_wkv4_forward_gated(g["w"], g["u"], g["k"], g["v"], r_open, checkpoints=True)
    y, ck0 = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], checkpoints=True)
    assert torch.equal(o, y) and torch.equal(ck, ck0)
    gk, gv, gr, gw, gu = rw.rwkv_wkv4_backward_gated(g["w"], g["u"], g["k"], g["v"], r_open, g["go"], ckpt=ck)
    gk0, gv0, gw0, gu0 = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["go"], ckpt=ck0)
    for a, b in ((gk, gk0), (gv, gv0), (gw, gw0), (gu, gu0)):
        assert torch.equal(a, b)
    assert float(gr.abs().max()) == 0.0


def test_gated_bf16_io(cuda_device):
    B, T, C = 2, 300, 64
    p = wi.wkv4_problem(B, T, C, 36, with_gy=True, gated=True, dtype=torch.bfloat16)
    g = _cuda(p, cuda_device)
    o, ck = rw.rwkv_wkv4_forward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], checkpoints=True)
    assert_close_rms(o, oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], p["r"]), TOL_BF16, "o bf16")
    got = rw.rwkv_wkv4_backward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], g["go"], ckpt=ck)
    ref = oracle.wkv4_gated_backward(p["w"], p["u"], p["k"], p["v"], p["r"], p["go"])
    for a, b, name in zip(got, ref, ("gk", "gv", "gr", "gw", "gu")):
        assert_close_rms(a, b, TOL_BF16, name + " bf16")


def test_gated_training_workload_full_size(cuda_device):
    # 8 x 4096 x 2048 with 1 % key outliers, r, go ~ N(0, 1): the launch configuration the
    # benchmark times; every output of 32 sampled channels (all batch rows) against the oracle
    B, T, C = 8, 4096, 2048
    p = wi.wkv4_problem(B, T, C, SEED + 2, outliers=True, with_gy=True, gated=True)
    g = _cuda(p, cuda_device)
    o, ck = rw.rwkv_wkv4_forward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], checkpoints=True)
    gk, gv, gr, gw, gu = rw.rwkv_wkv4_backward_gated(g["w"], g["u"], g["k"], g["v"], g["r"], g["go"], ckpt=ck)
    rw.rwkv_check_device_error()
    chans = torch.from_numpy(np.random.default_rng(3).choice(C, 32, replace=False))
    sub = {k: (v[:, :, chans] if v.dim() == 3 else v[chans]) for k, v in p.items()}
    cg = chans.to(cuda_device)
    assert_close_abs1(o[:, :, cg], oracle.wkv4_gated_forward(sub["w"], sub["u"], sub["k"], sub["v"], sub["r"]),
                      TOL_Y, "o")
    ref = oracle.wkv4_gated_backward(sub["w"], sub["u"], sub["k"], sub["v"], sub["r"], sub["go"])
    _check_grads((gk[:, :, cg], gv[:, :, cg], gr[:, :, cg], gw[cg], gu[cg]), ref)
