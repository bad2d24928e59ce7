"""GPU parity of the RWKV-4 WKV kernels against the fp64 oracle, through the
C-ABI (the Python binding only marshals pointers).  Tolerances: tests/_parity.py.

Shapes: the workloads' own sizes (1x64x128; 8x1024x768 with 1 % +-U(20,40) key
outliers; 8x4096x2048 forward+backward; 4096 streams x 4096 channels decode)
plus ragged cases that span several 32-channel tiles and a partial time tile."""
import numpy as np
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import (TOL_BF16, TOL_GRAD, TOL_Y, assert_close_abs1, assert_close_rms, assert_grads_close,
                     assert_state_close, wkv4_input_sensitivity)

pytestmark = pytest.mark.gpu
SEED = wi.CONFIG_SEED_BASE
ALGOS = [rw.ALGO_SEQUENTIAL, rw.ALGO_CHUNKED]


def _cuda(p, dev):
    return {k: v.to(dev) for k, v in p.items()}


@pytest.mark.parametrize("algo", ALGOS)
def test_forward_small_workload(cuda_device, algo):
    # 1 x 64 x 128, w log-uniform [0.01, 5], u ~ U(-1, 1), k, v ~ N(0, 1)
    p = wi.wkv4_problem(1, 64, 128, SEED + 0)
    y = rw.rwkv_wkv4_forward(**_cuda(p, cuda_device), algo=algo)
    ref = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    assert_close_abs1(y, ref, TOL_Y, "y")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("shape", [(3, 333, 100), (1, 1, 32), (2, 7, 4), (5, 250, 36)])
def test_forward_ragged(cuda_device, algo, shape):
    B, T, C = shape
    p = wi.wkv4_problem(B, T, C, 7, outliers=True)
    y, st = rw.rwkv_wkv4_forward(**_cuda(p, cuda_device), algo=algo, return_state=True)
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)
    assert_close_abs1(y, ref, TOL_Y, "y")
    assert_state_close(st, ref_st)


@pytest.mark.parametrize("algo", [rw.ALGO_AUTO] + ALGOS)
def test_forward_outlier_workload_full(cuda_device, algo):
    # 8 x 1024 x 768 with 1 % of keys replaced by +-U(20, 40): every element checked
    p = wi.wkv4_problem(8, 1024, 768, SEED + 1, outliers=True)
    y, st = rw.rwkv_wkv4_forward(**_cuda(p, cuda_device), algo=algo, return_state=True)
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)
    assert_close_abs1(y, ref, TOL_Y, "y")
    assert_state_close(st, ref_st)


def test_forward_few_channels_long_sequence(cuda_device):
    # 1 x 4096 x 768 (24 channel tiles): AUTO cuts time into segments; every element checked
    p = wi.wkv4_problem(1, 4096, 768, SEED + 1, outliers=True)
    assert rw.lib().rwkv_wkv4_forward_workspace_bytes(1, 4096, 768, rw.ALGO_AUTO) > 0
    y, st = rw.rwkv_wkv4_forward(**_cuda(p, cuda_device), algo=rw.ALGO_AUTO, return_state=True)
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)
    assert_close_abs1(y, ref, TOL_Y, "y")
    assert_state_close(st, ref_st)


@pytest.mark.parametrize("shape", [(1, 4096, 32), (1, 20001, 40), (2, 9000, 32)])
@pytest.mark.parametrize("with_state", [False, True])
def test_forward_many_segments(cuda_device, shape, with_state):
    # One or two lane tiles over a long sequence: the chunked schedule cuts it into 64 to 157
    # segments of one or two 64-step tiles (one launch, every tile resident), so a segment waits
    # for and folds up to 156 earlier summaries, more than the 32 polled at once; the last
    # segment is partial in the two ragged cases
    B, T, C = shape
    p = wi.wkv4_problem(B, T, C, SEED + 2, outliers=True)
    s_in = None
    if with_state:
        _, s_in = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :300], p["v"][:, :300], return_state=True)
    g = _cuda(p, cuda_device)
    st_dev = None
    if s_in is not None:
        st_dev = torch.zeros(3, B, C, dtype=torch.float32)
        st_dev[0], st_dev[1] = torch.from_numpy(s_in[0]).float(), torch.from_numpy(s_in[1]).float()
        st_dev = st_dev.to(cuda_device)
    y, st = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], st_dev, algo=rw.ALGO_CHUNKED, return_state=True)
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], state_in=s_in, return_state=True)
    assert_close_abs1(y, ref, TOL_Y, "y")
    assert_state_close(st, ref_st)


@pytest.mark.parametrize("shape", [(1, 20001, 40), (8, 1024, 768)])
def test_forward_chunked_state_in_place(cuda_device, shape):
    # state_out is state_in on the chunked schedule: the final state is written while other
    # segments fold the start state into theirs, so each must have read it first
    B, T, C = shape
    p = wi.wkv4_problem(B, T, C, SEED + 3, outliers=True)
    _, s_ref = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :100], p["v"][:, :100], return_state=True)
    st = torch.zeros(3, B, C, dtype=torch.float32)
    st[0], st[1] = torch.from_numpy(s_ref[0]).float(), torch.from_numpy(s_ref[1]).float()
    g = _cuda(p, cuda_device)
    st = st.to(cuda_device)
    h = rw.lib()
    wsb = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, rw.ALGO_CHUNKED))
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device=cuda_device)
    y = torch.empty(B, T, C, device=cuda_device)
    assert h.rwkv_wkv4_forward(B, T, C, rw.F32, rw._ptr(g["w"]), rw._ptr(g["u"]), rw._ptr(g["k"]), rw._ptr(g["v"]),
                               rw._ptr(y), rw._ptr(st), rw._ptr(st), None, 16, rw.ALGO_CHUNKED, rw._ptr(ws), wsb,
                               rw._stream(None)) == 0
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], state_in=s_ref, return_state=True)
    assert_close_abs1(y, ref, TOL_Y, "y")
    assert_state_close(st, ref_st)


def test_forward_single_large_outlier_slow_decay(cuda_device):
    # One +40 key at t = 1 and w = 0.01: the outlier dominates the state for
    # hundreds of steps, the case where per-step rounding of a running-max
    # exponent would drift.
    B, T, C = 2, 1024, 64
    p = wi.wkv4_problem(B, T, C, 11)
    p["k"][:, 1, :] = 40.0
    p["w"][:] = 0.01
    y = rw.rwkv_wkv4_forward(**_cuda(p, cuda_device))
    ref = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    assert_close_abs1(y, ref, TOL_Y, "y")


@pytest.mark.parametrize("algo", ALGOS)
def test_forward_split_sequence_resume(cuda_device, algo):
    B, T, C, cut = 2, 700, 64, 333
    p = wi.wkv4_problem(B, T, C, 12, outliers=True)
    g = _cuda(p, cuda_device)
    y1, s1 = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"][:, :cut].contiguous(), g["v"][:, :cut].contiguous(),
                                  algo=algo, return_state=True)
    y2, s2 = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"][:, cut:].contiguous(), g["v"][:, cut:].contiguous(),
                                  s1, algo=algo, return_state=True)
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)
    assert_close_abs1(torch.cat([y1, y2], 1), ref, TOL_Y, "y")
    assert_state_close(s2, ref_st)


def test_forward_state_in_place_and_external_state(cuda_device):
    B, T, C = 2, 50, 32
    p = wi.wkv4_problem(B, T, C, 13)
    _, s_ref = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :20], p["v"][:, :20], return_state=True)
    # an fp64 (A, B) state handed over as (A, B, 0)
    st = torch.zeros(3, B, C, dtype=torch.float32)
    st[0], st[1] = torch.from_numpy(s_ref[0]).float(), torch.from_numpy(s_ref[1]).float()
    g = _cuda(p, cuda_device)
    st = st.to(cuda_device)
    h = rw.lib()
    y = torch.empty(B, T - 20, C, device=cuda_device)
    k2, v2 = g["k"][:, 20:].contiguous(), g["v"][:, 20:].contiguous()
    assert h.rwkv_wkv4_forward(B, T - 20, C, rw.F32, rw._ptr(g["w"]), rw._ptr(g["u"]), rw._ptr(k2), rw._ptr(v2),
                               rw._ptr(y), rw._ptr(st), rw._ptr(st), None, 16, rw.ALGO_SEQUENTIAL, None, 0,
                               rw._stream(None)) == 0
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, 20:], p["v"][:, 20:], state_in=s_ref,
                                      return_state=True)
    assert_close_abs1(y, ref, TOL_Y, "y")
    assert_state_close(st, ref_st)  # state_out aliased state_in


@pytest.mark.parametrize("algo", ALGOS)
def test_forward_checkpoints_are_states(cuda_device, algo):
    B, T, C = 2, 100, 64
    p = wi.wkv4_problem(B, T, C, 14, outliers=True)
    _, ck = rw.rwkv_wkv4_forward(**_cuda(p, cuda_device), checkpoints=True, algo=algo)
    assert ck.shape == (7, 3, B, C)
    for j in range(1, 7):
        _, s = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :16 * j], p["v"][:, :16 * j], return_state=True)
        assert_state_close(ck[j], s, f"ckpt[{j}]")
    assert torch.all(ck[0, :2] == 0)


def test_forward_zero_length(cuda_device):
    B, C = 2, 64
    p = wi.wkv4_problem(B, 1, C, 15)
    g = _cuda(p, cuda_device)
    st_in = torch.randn(3, B, C, device=cuda_device).abs()
    st_out = torch.empty_like(st_in)
    k0 = torch.empty(B, 0, C, device=cuda_device)
    h = rw.lib()
    assert h.rwkv_wkv4_forward(B, 0, C, rw.F32, rw._ptr(g["w"]), rw._ptr(g["u"]), rw._ptr(k0), rw._ptr(k0),
                               rw._ptr(k0), rw._ptr(st_in), rw._ptr(st_out), None, 16, 0, None, 0,
                               rw._stream(None)) == 0
    torch.cuda.synchronize()
    assert torch.equal(st_in, st_out)


@pytest.mark.parametrize("use_ckpt", [True, False])
@pytest.mark.parametrize("shape", [(2, 100, 64), (3, 37, 100), (1, 16, 32)])
def test_backward_small(cuda_device, use_ckpt, shape):
    B, T, C = shape
    p = wi.wkv4_problem(B, T, C, 16, outliers=True, with_gy=True)
    g = _cuda(p, cuda_device)
    y, ck = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], checkpoints=True)
    gk, gv, gw, gu = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"],
                                           ckpt=ck if use_ckpt else None)
    r = oracle.wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["gy"])
    assert_grads_close((gk, gv, gw, gu), r)


def test_backward_with_initial_state(cuda_device):
    B, T, C = 2, 90, 64
    p = wi.wkv4_problem(B, T + 30, C, 17, outliers=True, with_gy=True)
    _, s0 = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :30], p["v"][:, :30], return_state=True)
    st = torch.zeros(3, B, C)
    st[0], st[1] = torch.from_numpy(s0[0]).float(), torch.from_numpy(s0[1]).float()
    q = {k: (v[:, 30:].contiguous() if v.dim() == 3 else v) for k, v in p.items()}
    g = _cuda(q, cuda_device)
    stg = st.to(cuda_device)
    _, ck = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], stg, checkpoints=True)
    out_ck = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], ckpt=ck)
    out_re = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], state_in=stg)
    r = oracle.wkv4_backward(q["w"], q["u"], q["k"], q["v"], q["gy"], state_in=st.double().numpy()[:2])
    for out in (out_ck, out_re):
        assert_grads_close(out, r)


def test_backward_deterministic(cuda_device):
    p = wi.wkv4_problem(4, 200, 128, 18, outliers=True, with_gy=True)
    g = _cuda(p, cuda_device)
    _, ck = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], checkpoints=True)
    a = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], ckpt=ck)
    b = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], ckpt=ck)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_training_workload_full_size(cuda_device):
    # 8 x 4096 x 2048, keys with 1 % outliers, gy ~ N(0, 1): forward + backward
    # in the launch configuration the benchmark times; every output element
    # (y, gk, gv over all 2048 channels and 8 batch rows, gw and gu per channel)
    # checked against the fp64 oracle over the whole problem.
    B, T, C = 8, 4096, 2048
    p = wi.wkv4_problem(B, T, C, SEED + 2, outliers=True, with_gy=True)
    g = _cuda(p, cuda_device)
    y, ck = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], checkpoints=True)
    gk, gv, gw, gu = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], ckpt=ck)
    rw.rwkv_check_device_error()
    del ck, g
    ref_y = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    assert_close_abs1(y, ref_y, TOL_Y, "y")
    del ref_y, y
    r = oracle.wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["gy"])
    # gw and gu entries are sums over 32,768 terms; where one is small beside its terms, half-ulp
    # perturbations of the fp32 inputs move the exact result by more than 1e-4 (the oracle shows it)
    floor = wkv4_input_sensitivity(oracle, p["w"], p["u"], p["k"], p["v"], p["gy"])
    rep = assert_grads_close((gk, gv, gw, gu), r, floor=floor)
    assert rep["gw_on_floor"] <= C // 8 and rep["gu_on_floor"] <= C // 8, rep
    # properties that hold for every lane: sum_t gk = 0 and sum_t gv = sum_t gy
    # (fp32 sums of 4096 terms: compared against the sum of magnitudes)
    sk = gk.double().sum(1)
    assert torch.all(sk.abs() <= 1e-4 * gk.double().abs().sum(1) + 1e-4)
    sv = gv.double().sum(1) - p["gy"].to(gv.device).double().sum(1)
    assert torch.all(sv.abs() <= 1e-4 * gv.double().abs().sum(1) + 1e-4)


def test_bf16_io(cuda_device):
    B, T, C = 2, 200, 64
    p = wi.wkv4_problem(B, T, C, 19, outliers=True, with_gy=True, dtype=torch.bfloat16)
    g = _cuda(p, cuda_device)
    y, ck = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], checkpoints=True)
    assert y.dtype == torch.bfloat16
    ref_y = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    assert_close_rms(y, ref_y, TOL_BF16, "y bf16")
    gk, gv, gw, gu = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], ckpt=ck)
    r = oracle.wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["gy"])
    for got, ref, name in zip((gk, gv, gw, gu), r, ("gk", "gv", "gw", "gu")):
        assert_close_rms(got, ref, TOL_BF16, name + " bf16")
    # decode step in bf16
    st = torch.zeros(3, B, C, device=cuda_device)
    ys = [rw.rwkv_wkv4_step(g["w"], g["u"], g["k"][:, t].contiguous(), g["v"][:, t].contiguous(), st)
          for t in range(20)]
    assert_close_rms(torch.stack(ys, 1), ref_y[:, :20], TOL_BF16, "step bf16")


def test_step_matches_forward_small(cuda_device):
    B, C, T0, T1 = 64, 256, 128, 256
    p = wi.wkv4_problem(B, T0 + T1, C, 20, outliers=True)
    g = _cuda(p, cuda_device)
    _, st = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"][:, :T0].contiguous(), g["v"][:, :T0].contiguous(),
                                 return_state=True)
    ys = []
    for t in range(T0, T0 + T1):
        ys.append(rw.rwkv_wkv4_step(g["w"], g["u"], g["k"][:, t].contiguous(), g["v"][:, t].contiguous(), st))
    ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)
    assert_close_abs1(torch.stack(ys, 1), ref[:, T0:], TOL_Y, "decode y")
    assert_state_close(st, ref_st)
    # scalar path: C not a multiple of 4, separate in/out state
    q = wi.wkv4_problem(3, 40, 10, 21)
    gq = _cuda(q, cuda_device)
    s_in = torch.zeros(3, 3, 10, device=cuda_device)
    out = []
    for t in range(40):
        s_out = torch.empty_like(s_in)
        out.append(rw.rwkv_wkv4_step(gq["w"], gq["u"], gq["k"][:, t].contiguous(), gq["v"][:, t].contiguous(),
                                     s_in, state_out=s_out))
        s_in = s_out
    assert_close_abs1(torch.stack(out, 1), oracle.wkv4_forward(q["w"], q["u"], q["k"], q["v"]), TOL_Y, "y")


def test_decode_workload_full_size(cuda_device):
    # 4096 independent streams x 4096 channels: a 128-token N(0,1) prefix by the
    # forward's state_out, then 256 decode steps with state in/out each step.
    # Every decode output is checked against the time-parallel forward over the
    # same 384 tokens (all streams), and 16 sampled streams against the oracle.
    B, C, T0, T1 = 4096, 4096, 128, 256
    T = T0 + T1
    dev = cuda_device
    seed = SEED + 3
    w, u = wi.wkv4_params(seed, C, device=dev)
    kp = wi.btc_field("k", seed, B, T, C, t0=0, t1=T0, device=dev)
    vp = wi.btc_field("v", seed, B, T, C, t0=0, t1=T0, device=dev)
    _, st = rw.rwkv_wkv4_forward(w, u, kp, vp, return_state=True)
    samp = torch.from_numpy(np.random.default_rng(3).choice(B, 16, replace=False)).to(dev)
    ks, vs = [kp[samp].cpu()], [vp[samp].cpu()]
    del kp, vp
    ydec = torch.empty(B, T1, C, device=dev)
    for i, t in enumerate(range(T0, T)):
        kt = wi.btc_field("k", seed, B, T, C, t0=t, t1=t + 1, device=dev)[:, 0].contiguous()
        vt = wi.btc_field("v", seed, B, T, C, t0=t, t1=t + 1, device=dev)[:, 0].contiguous()
        ydec[:, i] = rw.rwkv_wkv4_step(w, u, kt, vt, st)
        ks.append(kt[samp].unsqueeze(1).cpu())
        vs.append(vt[samp].unsqueeze(1).cpu())
    # oracle on sampled streams (inputs are the bytes the GPU consumed)
    ref = oracle.wkv4_forward(w.cpu(), u.cpu(), torch.cat(ks, 1), torch.cat(vs, 1))
    assert_close_abs1(ydec[samp], ref[:, T0:], TOL_Y, "decode vs oracle")
    # GPU time-parallel forward over the same 384 tokens, 512 streams at a time
    worst = 0.0
    for b0 in range(0, B, 512):
        k = wi.btc_field("k", seed, B, T, C, b0=b0, b1=b0 + 512, device=dev)
        v = wi.btc_field("v", seed, B, T, C, b0=b0, b1=b0 + 512, device=dev)
        y = rw.rwkv_wkv4_forward(w, u, k, v)
        d = (y[:, T0:] - ydec[b0:b0 + 512]).abs() / torch.clamp(y[:, T0:].abs(), min=1.0)
        worst = max(worst, d.max().item())
        del k, v, y, d
    assert worst <= 2 * TOL_Y, worst


def test_workspace_and_alignment_errors(cuda_device):
    p = _cuda(wi.wkv4_problem(8, 1024, 768, 22), cuda_device)
    h = rw.lib()
    y = torch.empty_like(p["k"])
    args = (8, 1024, 768, rw.F32, rw._ptr(p["w"]), rw._ptr(p["u"]), rw._ptr(p["k"]), rw._ptr(p["v"]),
            rw._ptr(y), None, None, None, 16, rw.ALGO_CHUNKED)
    need = h.rwkv_wkv4_forward_workspace_bytes(8, 1024, 768, rw.ALGO_CHUNKED)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    assert h.rwkv_wkv4_forward(*args, rw._ptr(ws), need - 4, rw._stream(None)) == 3
    assert h.rwkv_wkv4_forward(*args, rw._ptr(ws), need, rw._stream(None)) == 0
    # k off 16-byte alignment: the plain-access instance serves it, with the TMA path's arithmetic
    kk = torch.empty(8 * 1024 * 768 + 1, device=cuda_device)[1:].view(8, 1024, 768)
    kk.copy_(p["k"])
    y_plain = torch.empty_like(y)
    assert h.rwkv_wkv4_forward(8, 1024, 768, rw.F32, rw._ptr(p["w"]), rw._ptr(p["u"]), rw._ptr(kk),
                               rw._ptr(p["v"]), rw._ptr(y_plain), None, None, None, 16, 1, None, 0,
                               rw._stream(None)) == 0
    y_tma = torch.empty_like(y)
    assert h.rwkv_wkv4_forward(8, 1024, 768, rw.F32, rw._ptr(p["w"]), rw._ptr(p["u"]), rw._ptr(p["k"]),
                               rw._ptr(p["v"]), rw._ptr(y_tma), None, None, None, 16, 1, None, 0,
                               rw._stream(None)) == 0
    rw.rwkv_check_device_error()
    assert torch.equal(y_plain, y_tma)
