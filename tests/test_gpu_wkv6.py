"""GPU parity of the Finch / RWKV-6 WKV forward (per-token decay) and its
decode step against the fp64 oracle, through the C-ABI.  bf16 inputs are
widened exactly for the oracle; omega is fp32 on both sides.
Tolerance for the bf16 output y and the fp32 final state alike:
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


def _ref(p, s_in=None):
    return oracle.wkv6_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], s_in=s_in, return_state=True)


@pytest.mark.parametrize("shape", [(1, 64, 1), (1, 100, 2), (2, 33, 3), (1, 1, 1), (2, 200, 3)])
def test_forward_small(cuda_device, shape):
    B, T, H = shape
    p = wi.wkv6_problem(B, T, H, 64, seed=40)
    y, s = rw.rwkv_wkv6_forward(**_cuda(p, cuda_device), return_state=True)
    ref, ref_s = _ref(p)
    assert_close_rms(y, ref, TOL_BF16, "y")
    assert_close_rms(s, ref_s, TOL_BF16, "s_out")


@pytest.mark.parametrize("omega_range", [(-6.0, 0.0), (-3.0, 0.9), (-1.0, 2.0)])
def test_forward_decay_ranges(cuda_device, omega_range):
    # (-6, 0): every chunk on the tensor cores; (-1, 2): every chunk decays too fast in some channel
    # and takes the per-token recurrence; (-3, 0.9): the half-chunk log-decay straddles the limit of
    # the factorization, so chunks of both kinds alternate on one state.
    p = wi.wkv6_problem(2, 300, 3, 64, seed=41, omega_range=omega_range)
    y, s = rw.rwkv_wkv6_forward(**_cuda(p, cuda_device), return_state=True)
    ref, ref_s = _ref(p)
    assert_close_rms(y, ref, TOL_BF16, "y")
    assert_close_rms(s, ref_s, TOL_BF16, "s_out")


def test_zero_decay_tokens(cuda_device):
    # omega = 8 at a few tokens (w = exp(-e^8) = 0: the state is erased there), including the
    # first and the last token of a chunk; the chunks holding them take the recurrence.
    B, T, H = 2, 256, 2
    p = wi.wkv6_problem(B, T, H, 64, seed=42)
    for t in (5, 63, 64, 130, 255):
        p["omega"][:, t] = 8.0
    y, s = rw.rwkv_wkv6_forward(**_cuda(p, cuda_device), return_state=True)
    ref, ref_s = _ref(p)
    assert_close_rms(y, ref, TOL_BF16, "y")
    assert_close_rms(s, ref_s, TOL_BF16, "s_out")


def test_constant_decay_matches_eagle_oracle(cuda_device):
    # omega_t constant in time: the Eagle recurrence (pinned separately) gives the same result.
    B, T, H = 2, 150, 2
    q = wi.wkv5_problem(B, T, H, 64, seed=43)
    om_t = q["omega"][None, None].expand(B, T, H, 64).contiguous()
    y, s = rw.rwkv_wkv6_forward(q["r"].to(cuda_device), q["k"].to(cuda_device), q["v"].to(cuda_device),
                                om_t.to(cuda_device), q["u"].to(cuda_device), return_state=True)
    ref, ref_s = oracle.wkv5_forward(q["r"], q["k"], q["v"], q["omega"], q["u"], return_state=True)
    assert_close_rms(y, ref, TOL_BF16, "y")
    assert_close_rms(s, ref_s, TOL_BF16, "s_out")


def test_forward_split_state(cuda_device):
    B, T, H, cut = 2, 170, 2, 77
    p = wi.wkv6_problem(B, T, H, 64, seed=44)
    g = _cuda(p, cuda_device)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    y1, s1 = rw.rwkv_wkv6_forward(sl(g["r"], 0, cut), sl(g["k"], 0, cut), sl(g["v"], 0, cut),
                                  sl(g["omega"], 0, cut), g["u"], return_state=True)
    y2, s2 = rw.rwkv_wkv6_forward(sl(g["r"], cut, T), sl(g["k"], cut, T), sl(g["v"], cut, T),
                                  sl(g["omega"], cut, T), g["u"], s1, return_state=True)
    ref, ref_s = _ref(p)
    assert_close_rms(torch.cat([y1, y2], 1), ref, TOL_BF16, "y")
    assert_close_rms(s2, ref_s, TOL_BF16, "s_out")


def test_state_in_place(cuda_device):
    B, T, H = 1, 90, 2
    p = wi.wkv6_problem(B, T, H, 64, seed=45)
    g = _cuda(p, cuda_device)
    s0 = torch.from_numpy(_ref(wi.wkv6_problem(B, 20, H, 64, seed=46))[1]).float().to(cuda_device)
    y1, s1 = rw.rwkv_wkv6_forward(**g, s_in=s0, return_state=True)
    s_io = s0.clone()
    h = rw.lib()
    y2 = torch.empty_like(y1)
    wsb = int(h.rwkv_wkv6_forward_workspace_bytes(B, T, H, 64))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=cuda_device)
    assert h.rwkv_wkv6_forward(B, T, H, 64, g["r"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(),
                               g["omega"].data_ptr(), g["u"].data_ptr(), y2.data_ptr(), s_io.data_ptr(),
                               s_io.data_ptr(), ws.data_ptr(), wsb, None) == 0
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(s1, s_io)
    ref, ref_s = _ref(p, s_in=s0.cpu().double().numpy())
    assert_close_rms(y1, ref, TOL_BF16, "y")
    assert_close_rms(s1, ref_s, TOL_BF16, "s_out")


def test_finch_workload_full_size(cuda_device):
    # B4 T4096 H40 N64 with per-token omega = U(-6, 0) base + 0.5 N(0, 1): the whole
    # output and final state of all 160 (b, h) heads checked element by element.
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv6_problem(B, T, H, N, seed=SEED + 6)
    y, s = rw.rwkv_wkv6_forward(**_cuda(p, cuda_device), return_state=True)
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv6_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    yc, sc = y.cpu(), s.cpu()
    for b in range(B):
        for h in range(H):  # the rms of each rule is taken per head
            assert_close_rms(yc[b, :, h], ref[b, :, h], TOL_BF16, f"y head ({b},{h})")
            assert_close_rms(sc[b, h], ref_s[b, h], TOL_BF16, f"s head ({b},{h})")


def test_finch_fast_decay_full_size(cuda_device):
    # B4 T4096 H40 N64 with per-token omega = U(-1, 2) base + 0.5 N(0, 1): nearly
    # every chunk decays too fast for the factorization and runs by the recurrence;
    # all 160 heads checked element by element
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv6_problem(B, T, H, N, seed=SEED + 7, omega_range=(-1.0, 2.0))
    y, s = rw.rwkv_wkv6_forward(**_cuda(p, cuda_device), return_state=True)
    rw.rwkv_check_device_error()
    ref, ref_s = oracle.wkv6_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    yc, sc = y.cpu(), s.cpu()
    for b in range(B):
        for h in range(H):
            assert_close_rms(yc[b, :, h], ref[b, :, h], TOL_BF16, f"y head ({b},{h})")
            assert_close_rms(sc[b, h], ref_s[b, h], TOL_BF16, f"s head ({b},{h})")


# ------------------------------------------------------------------ decode step
def _token(p, t):
    return {n: p[n][:, t].contiguous() for n in ("r", "k", "v", "omega")}


def test_step_matches_oracle(cuda_device):
    B, H, t0 = 3, 5, 20
    p = wi.wkv6_problem(B, t0 + 1, H, 64, seed=47)
    _, s0 = oracle.wkv6_forward(p["r"][:, :t0], p["k"][:, :t0], p["v"][:, :t0], p["omega"][:, :t0], p["u"],
                                return_state=True)
    s0 = torch.from_numpy(s0).float()
    tok = _token(p, t0)
    y, s1 = rw.rwkv_wkv6_step(**_cuda(tok, cuda_device), u=p["u"].to(cuda_device), state=s0.to(cuda_device))
    ref, ref_s = oracle.wkv6_forward(*(tok[n][:, None] for n in ("r", "k", "v", "omega")), p["u"],
                                     s0.double().numpy(), return_state=True)
    assert_close_rms(y, ref[:, 0], TOL_BF16, "y")
    assert_close_rms(s1, ref_s, TOL_BF16, "s_out")


@pytest.mark.parametrize("omega_range", [(-6.0, 0.0), (-1.0, 2.0)])
def test_step_sequence_matches_forward_oracle(cuda_device, omega_range):
    B, T, H = 2, 40, 3
    p = wi.wkv6_problem(B, T, H, 64, seed=48, omega_range=omega_range)
    g = _cuda(p, cuda_device)
    state = torch.zeros(B, H, 64, 64, device=cuda_device)
    ys = []
    for t in range(T):
        y, _ = rw.rwkv_wkv6_step(**_token(g, t), u=g["u"], state=None if t == 0 else state, state_out=state)
        ys.append(y)
    ref, ref_s = _ref(p)
    assert_close_rms(torch.stack(ys, 1), ref, TOL_BF16, "y")
    assert_close_rms(state, ref_s, TOL_BF16, "state")


def test_step_continues_the_forward(cuda_device):
    # forward over 100 tokens, then 28 decode steps from its state: the oracle over all 128 tokens
    B, T, H, T1 = 2, 128, 4, 100
    p = wi.wkv6_problem(B, T, H, 64, seed=49)
    g = _cuda(p, cuda_device)
    sl = lambda x: x[:, :T1].contiguous()
    y1, state = rw.rwkv_wkv6_forward(sl(g["r"]), sl(g["k"]), sl(g["v"]), sl(g["omega"]), g["u"],
                                     return_state=True)
    ys = [y1]
    for t in range(T1, T):
        y, _ = rw.rwkv_wkv6_step(**_token(g, t), u=g["u"], state=state, state_out=state)
        ys.append(y[:, None])
    ref, ref_s = _ref(p)
    assert_close_rms(torch.cat(ys, 1), ref, TOL_BF16, "y")
    assert_close_rms(state, ref_s, TOL_BF16, "state")
