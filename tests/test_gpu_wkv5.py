"""GPU parity of the Eagle / RWKV-5 matrix-state WKV forward and decode step
against the fp64 oracle, through the C-ABI.  bf16 inputs are widened exactly for the oracle.
Tolerance for the bf16 output y and for the fp32 final state alike:
|got - ref| <= 8e-3 * max(|ref|, rms(ref))."""
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import TOL_BF16, assert_close_rms

pytestmark = pytest.mark.gpu
SEED = wi.CONFIG_SEED_BASE


def _cuda(p, dev):
    return {k: v.to(dev) for k, v in p.items()}


@pytest.mark.parametrize("shape", [(1, 64, 1), (1, 100, 2), (2, 33, 3), (1, 1, 1), (2, 200, 3)])
def test_forward_small(cuda_device, shape):
    B, T, H = shape
    p = wi.wkv5_problem(B, T, H, 64, seed=30)
    y, s = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), return_state=True)
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    assert_close_rms(y, ref, TOL_BF16, "y")
    assert_close_rms(s, ref_s, TOL_BF16, "s_out")


@pytest.mark.parametrize("omega_range", [(-1.0, 2.0), (-8.0, -4.0), (0.5, 0.9)])
def test_forward_decay_ranges(cuda_device, omega_range):
    # fast decays (exp(omega) > 2.5, w < 0.082) take the recurrent path inside
    # the kernel; slow and moderate decays the chunked tensor-core path
    p = wi.wkv5_problem(2, 150, 3, 64, seed=32, omega_range=omega_range)
    y, s = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), return_state=True)
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    assert_close_rms(y, ref, TOL_BF16, "y")
    assert_close_rms(s, ref_s, TOL_BF16, "s_out")


def test_forward_split_state(cuda_device):
    B, T, H, cut = 2, 150, 2, 61
    p = wi.wkv5_problem(B, T, H, 64, seed=31)
    g = _cuda(p, cuda_device)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    y1, s1 = rw.rwkv_wkv5_forward(sl(g["r"], 0, cut), sl(g["k"], 0, cut), sl(g["v"], 0, cut), g["omega"], g["u"],
                                  return_state=True)
    y2 = rw.rwkv_wkv5_forward(sl(g["r"], cut, T), sl(g["k"], cut, T), sl(g["v"], cut, T), g["omega"], g["u"],
                              s1)
    ref = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"])
    assert_close_rms(torch.cat([y1, y2], 1), ref, TOL_BF16, "y")


def test_eagle_workload_full_size(cuda_device):
    # B4 T4096 H40 N64, omega ~ U(-6, 0), u ~ U(-1, 1), zero initial state: the
    # whole output and final state of all 160 (b, h) heads checked element by element.
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv5_problem(B, T, H, N, seed=SEED + 4)
    y, s = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), return_state=True)
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    yc, sc = y.cpu(), s.cpu()
    for b in range(B):
        for h in range(H):  # the rms of each rule is taken per head
            assert_close_rms(yc[b, :, h], ref[b, :, h], TOL_BF16, f"y head ({b},{h})")
            assert_close_rms(sc[b, h], ref_s[b, h], TOL_BF16, f"s head ({b},{h})")


def test_forward_mixed_heads_with_state(cuda_device):
    # heads 1 and 3 decay fast in some channels (per-token recurrence on the CUDA
    # cores), the others slowly (chunked tensor-core path), in one launch, from a
    # nonzero state and split into two calls at a ragged token
    B, T, H, cut = 2, 230, 4, 77
    p = wi.wkv5_problem(B, T, H, 64, seed=33)
    fastp = wi.wkv5_problem(B, T, H, 64, seed=34, omega_range=(-1.0, 2.0))
    p["omega"][1] = fastp["omega"][1]
    p["omega"][3] = fastp["omega"][3]
    s0 = wi.wkv5_problem(B, 64, H, 64, seed=35)["r"].float()
    s0 = s0.permute(0, 2, 1, 3).contiguous()  # [B,H,64,64], values ~ N(0, 1/64)
    g = _cuda(p, cuda_device)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    y1, s1 = rw.rwkv_wkv5_forward(sl(g["r"], 0, cut), sl(g["k"], 0, cut), sl(g["v"], 0, cut), g["omega"], g["u"],
                                  s0.to(cuda_device), return_state=True)
    y2, s2 = rw.rwkv_wkv5_forward(sl(g["r"], cut, T), sl(g["k"], cut, T), sl(g["v"], cut, T), g["omega"], g["u"],
                                  s1, return_state=True)
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], s_in=s0.double().numpy(),
                                     return_state=True)
    yc, sc = torch.cat([y1, y2], 1).cpu(), s2.cpu()
    for b in range(B):
        for h in range(H):
            assert_close_rms(yc[b, :, h], ref[b, :, h], TOL_BF16, f"y head ({b},{h})")
            assert_close_rms(sc[b, h], ref_s[b, h], TOL_BF16, f"s head ({b},{h})")


def test_eagle_fast_decay_full_size(cuda_device):
    # B4 T4096 H40 N64 with omega ~ U(-1, 2): every head has channels with
    # w < 0.082 and runs by the recurrence; all 160 heads checked element by element
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv5_problem(B, T, H, N, seed=SEED + 5, omega_range=(-1.0, 2.0))
    y, s = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), return_state=True)
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    yc, sc = y.cpu(), s.cpu()
    for b in range(B):
        for h in range(H):
            assert_close_rms(yc[b, :, h], ref[b, :, h], TOL_BF16, f"y head ({b},{h})")
            assert_close_rms(sc[b, h], ref_s[b, h], TOL_BF16, f"s head ({b},{h})")


# ------------------------------------------------------------------ the slot plan
def _state(p, B, H, seed):
    """A state the recurrence produces: the oracle's after 64 other tokens with p's decays and
    bonus, rounded to fp32 (so its size matches the decays, as a state handed over would)."""
    q = wi.wkv5_problem(B, 64, H, 64, seed=seed)
    _, s = oracle.wkv5_forward(q["r"], q["k"], q["v"], p["omega"], p["u"], return_state=True)
    return torch.from_numpy(s).float()


def _check_heads(y, s, ref, ref_s):
    yc, sc = y.cpu(), s.cpu()
    for b in range(yc.shape[0]):
        for h in range(yc.shape[2]):
            assert_close_rms(yc[b, :, h], ref[b, :, h], TOL_BF16, f"y head ({b},{h})")
            assert_close_rms(sc[b, h], ref_s[b, h], TOL_BF16, f"s head ({b},{h})")


@pytest.mark.parametrize("shape,omega_range", [((4, 1000, 40), (-6.0, 0.0)), ((1, 700, 150), (-6.0, 0.0)),
                                               ((2, 333, 80), (-1.0, 2.0)), ((1, 200, 222), (-6.0, 0.0)),
                                               ((1, 1500, 3), (-6.0, 0.0)), ((8, 300, 40), (-1.0, 2.0)),
                                               ((1, 64 * 40 + 17, 1), (-1.0, 2.0))])
def test_forward_slot_plan(cuda_device, shape, omega_range):
    # The heads' chunks laid end to end and dealt out to 296 CTAs: a CTA holds the tail of one
    # head, whole heads and the start of another, and folds the summaries of the CTAs before it
    # into the start state of a head it does not start (one head over 41 CTAs, 3 heads over 8
    # to 9 each, 320 heads over two per CTA).  Every head against the oracle, from a nonzero
    # state, T ragged, slow and fast decays.
    B, T, H = shape
    assert rw.lib().rwkv_wkv5_forward_workspace_bytes(B, T, H, 64) > 0
    p = wi.wkv5_problem(B, T, H, 64, seed=36, omega_range=omega_range)
    s0 = _state(p, B, H, 37)
    y, s = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), s_in=s0.to(cuda_device), return_state=True)
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], s_in=s0.double().numpy(),
                                     return_state=True)
    _check_heads(y, s, ref, ref_s)
    y2, s2 = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), s_in=s0.to(cuda_device), return_state=True)
    assert torch.equal(y, y2) and torch.equal(s, s2)  # the summaries fold in a fixed order


def test_forward_slot_plan_state_in_place(cuda_device):
    # s_out is s_in: the CTA holding a head's last chunk writes its final state while the CTAs
    # holding its earlier chunks may still be running, so each reads s_in before it publishes
    # its summary
    B, T, H = 4, 1000, 40
    q = wi.wkv5_problem(B, T, H, 64, seed=38)
    p = _cuda(q, cuda_device)
    s0 = _state(q, B, H, 39)
    st = s0.to(cuda_device)
    h = rw.lib()
    wsb = int(h.rwkv_wkv5_forward_workspace_bytes(B, T, H, 64))
    ws = torch.empty(wsb, dtype=torch.uint8, device=cuda_device)
    y = torch.empty_like(p["r"])
    assert h.rwkv_wkv5_forward(B, T, H, 64, rw._ptr(p["r"]), rw._ptr(p["k"]), rw._ptr(p["v"]), rw._ptr(p["omega"]),
                               rw._ptr(p["u"]), rw._ptr(y), rw._ptr(st), rw._ptr(st), rw._ptr(ws), wsb,
                               rw._stream(None)) == 0
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv5_forward(q["r"], q["k"], q["v"], q["omega"], q["u"], s_in=s0.double().numpy(),
                                     return_state=True)
    _check_heads(y, st, ref, ref_s)


def test_forward_slot_plan_two_streams(cuda_device):
    # Two calls in flight at once on two streams, each with its own workspace: their CTAs share
    # the SMs (neither call's 296 CTAs are all resident), and a CTA waits only for CTAs of its own
    # call that have already started.  Both finish, and each equals its call run alone, bit for bit.
    B, T, H = 4, 600, 40
    g1 = _cuda(wi.wkv5_problem(B, T, H, 64, seed=51), cuda_device)
    g2 = _cuda(wi.wkv5_problem(B, T, H, 64, seed=52, omega_range=(-1.0, 2.0)), cuda_device)
    ref1, ref2 = rw.rwkv_wkv5_forward(**g1), rw.rwkv_wkv5_forward(**g2)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(device=cuda_device), torch.cuda.Stream(device=cuda_device)
    for _ in range(3):
        with torch.cuda.stream(s1):
            y1 = rw.rwkv_wkv5_forward(**g1, stream=s1)
        with torch.cuda.stream(s2):
            y2 = rw.rwkv_wkv5_forward(**g2, stream=s2)
        torch.cuda.synchronize()
        rw.rwkv_check_device_error()
        assert torch.equal(y1, ref1) and torch.equal(y2, ref2)


# ------------------------------------------------------------------ decode step
def _token(p, t):
    return {n: p[n][:, t].contiguous() for n in ("r", "k", "v")}


def _prefix_state(p, t0):
    """The oracle's fp64 state after the first t0 tokens of problem p, as fp32."""
    _, s = oracle.wkv5_forward(p["r"][:, :t0], p["k"][:, :t0], p["v"][:, :t0], p["omega"], p["u"],
                               return_state=True)
    return torch.from_numpy(s).float()


def test_step_matches_oracle(cuda_device):
    B, H, t0 = 3, 5, 20
    p = wi.wkv5_problem(B, t0 + 1, H, 64, seed=33)
    s0 = _prefix_state(p, t0)
    tok = _token(p, t0)
    y, s1 = rw.rwkv_wkv5_step(**_cuda(tok, cuda_device), omega=p["omega"].to(cuda_device),
                              u=p["u"].to(cuda_device), state=s0.to(cuda_device))
    ref, ref_s = oracle.wkv5_forward(tok["r"][:, None], tok["k"][:, None], tok["v"][:, None], p["omega"], p["u"],
                                     s0.double().numpy(), return_state=True)
    assert_close_rms(y, ref[:, 0], TOL_BF16, "y")
    assert_close_rms(s1, ref_s, TOL_BF16, "s_out")


@pytest.mark.parametrize("omega_range", [(-6.0, 0.0), (-1.0, 2.0)])
def test_step_sequence_matches_forward_oracle(cuda_device, omega_range):
    # T steps from a zero state, state updated in place, against the oracle's forward over the same tokens
    B, T, H = 2, 40, 3
    p = wi.wkv5_problem(B, T, H, 64, seed=34, omega_range=omega_range)
    g = _cuda(p, cuda_device)
    state = torch.zeros(B, H, 64, 64, device=cuda_device)
    ys = []
    for t in range(T):
        y, _ = rw.rwkv_wkv5_step(**_token(g, t), omega=g["omega"], u=g["u"], state=None if t == 0 else state,
                                 state_out=state)
        ys.append(y)
    ref, ref_s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    assert_close_rms(torch.stack(ys, 1), ref, TOL_BF16, "y")
    assert_close_rms(state, ref_s, TOL_BF16, "state")


def test_step_in_place_equals_out_of_place(cuda_device):
    B, H = 4, 6
    p = wi.wkv5_problem(B, 9, H, 64, seed=35)
    g = _cuda(p, cuda_device)
    s0 = _prefix_state(p, 8).to(cuda_device)
    tok = _token(g, 8)
    y1, s1 = rw.rwkv_wkv5_step(**tok, omega=g["omega"], u=g["u"], state=s0)
    s_in_place = s0.clone()
    y2, s2 = rw.rwkv_wkv5_step(**tok, omega=g["omega"], u=g["u"], state=s_in_place, state_out=s_in_place)
    assert torch.equal(y1, y2) and torch.equal(s1, s2) and s2.data_ptr() == s_in_place.data_ptr()


def test_step_workload_full_size(cuda_device):
    # the decode bench's shape: 512 streams x 40 heads x 64, one step from a state
    # reached after 16 tokens; every head checked
    B, H, t0 = 512, 40, 16
    p = wi.wkv5_problem(B, t0 + 1, H, 64, seed=SEED + 5)
    s0 = _prefix_state(p, t0)
    tok = _token(p, t0)
    y, s1 = rw.rwkv_wkv5_step(**_cuda(tok, cuda_device), omega=p["omega"].to(cuda_device),
                              u=p["u"].to(cuda_device), state=s0.to(cuda_device))
    ref, ref_s = oracle.wkv5_forward(tok["r"][:, None], tok["k"][:, None], tok["v"][:, None], p["omega"], p["u"],
                                     s0.double().numpy(), return_state=True)
    assert_close_rms(y, ref[:, 0], TOL_BF16, "y")
    assert_close_rms(s1, ref_s, TOL_BF16, "s_out")
