"""GPU parity of the Eagle / RWKV-5 matrix-state WKV forward against the fp64
oracle, through the C-ABI.  bf16 inputs are widened exactly for the oracle.
Tolerance for the bf16 output y and for the fp32 final state alike:
|got - ref| <= 8e-3 * max(|ref|, rms(ref))."""
import numpy as np
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
    # B4 T4096 H40 N64, omega ~ U(-6, 0), u ~ U(-1, 1), zero initial state:
    # whole output on the GPU, 12 sampled (b, h) heads checked element by element.
    B, T, H, N = 4, 4096, 40, 64
    p = wi.wkv5_problem(B, T, H, N, seed=SEED + 4)
    y, s = rw.rwkv_wkv5_forward(**_cuda(p, cuda_device), return_state=True)
    rng = np.random.default_rng(4)
    for b, h in zip(rng.integers(0, B, 12), rng.integers(0, H, 12)):
        sub = lambda x: x[b:b + 1, :, h:h + 1]
        ref, ref_s = oracle.wkv5_forward(sub(p["r"]), sub(p["k"]), sub(p["v"]), p["omega"][h:h + 1],
                                         p["u"][h:h + 1], return_state=True)
        assert_close_rms(y[b:b + 1, :, h:h + 1], ref, TOL_BF16, f"y head ({b},{h})")
        assert_close_rms(s[b:b + 1, h:h + 1], ref_s, TOL_BF16, f"s head ({b},{h})")
