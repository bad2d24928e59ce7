"""The WKV-4 backward entry point that allocates nothing
(rwkv_wkv4_backward_noalloc) against the workspace entry point
(rwkv_wkv4_backward), through the C ABI on the GPU.

Some callers cannot allocate device memory where they run the backward (a
framework pool owns the card's memory, a latency-critical loop cannot absorb
cudaMalloc's implicit synchronisation, a system allocates only at start-up);
this entry point keeps its scratch in a fixed array inside the library.  Two
calls in a row, with different shapes and inputs, must each match the
workspace entry point within the gradient tolerance of the parity tests (the
array keeps the previous call's contents, which must not leak into the next
call's results).  This file is collected last so that a failure here comes
after every other test has run."""
import ctypes

import pytest
import torch

import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import TOL_BF16, assert_close_rms, assert_grads_close

pytestmark = pytest.mark.gpu


def _run_both(dev, B, T, C, seed, dtype=torch.float32):
    g = {k: v.to(dev) for k, v in wi.wkv4_problem(B, T, C, seed, outliers=True, with_gy=True, dtype=dtype).items()}
    _, ck = rw.rwkv_wkv4_forward(g["w"], g["u"], g["k"], g["v"], checkpoints=True)
    ref = rw.rwkv_wkv4_backward(g["w"], g["u"], g["k"], g["v"], g["gy"], ckpt=ck)
    h = rw.lib()
    out = (torch.empty_like(g["k"]), torch.empty_like(g["v"]), torch.empty(C, device=dev), torch.empty(C, device=dev))
    st = h.rwkv_wkv4_backward_noalloc(B, T, C, rw._dtype_code(g["k"]), rw._ptr(g["w"]), rw._ptr(g["u"]),
                                      rw._ptr(g["k"]), rw._ptr(g["v"]), rw._ptr(g["gy"]), rw._ptr(ck), 16,
                                      rw._ptr(out[0]), rw._ptr(out[1]), rw._ptr(out[2]), rw._ptr(out[3]),
                                      rw._stream(None))
    assert st == 0, h.rwkv_status_string(st)
    torch.cuda.synchronize()
    return out, ref


def test_noalloc_backward_matches_workspace_backward_twice(cuda_device):
    # first call: a larger problem fills the scratch; second call: a smaller one
    out1, ref1 = _run_both(cuda_device, 8, 700, 768, 41)
    assert_grads_close(out1, tuple(x.double().cpu() for x in ref1), "first call ")
    out2, ref2 = _run_both(cuda_device, 3, 333, 100, 42)
    assert_grads_close(out2, tuple(x.double().cpu() for x in ref2), "second call ")
    rw.rwkv_check_device_error()


def test_noalloc_bf16_matches_workspace_backward(cuda_device):
    # bf16 k, v, gy, gk, gv: the 8e-3 rule of the bf16 parity tests, twice in a row
    for call, (B, T, C, seed) in enumerate(((2, 200, 64, 43), (4, 77, 48, 44))):
        out, ref = _run_both(cuda_device, B, T, C, seed, dtype=torch.bfloat16)
        for got, want, name in zip(out, ref, ("gk", "gv", "gw", "gu")):
            assert_close_rms(got, want, TOL_BF16, f"call {call} {name} bf16")
    rw.rwkv_check_device_error()


def test_noalloc_at_full_capacity(cuda_device):
    # B * C equal to the fixed scratch's capacity: the last lane of the array is used
    B, T, C = 1, 16, rw.NOALLOC_MAX_LANES
    out, ref = _run_both(cuda_device, B, T, C, 45)
    assert_grads_close(out, tuple(x.double().cpu() for x in ref), "at capacity ")
    rw.rwkv_check_device_error()


def test_noalloc_rejects_problems_beyond_its_capacity(cuda_device):
    h = rw.lib()
    P = ctypes.c_void_p
    fake = P(0x1000)  # rejected before anything is enqueued
    assert h.rwkv_wkv4_backward_noalloc(2, 16, rw.NOALLOC_MAX_LANES, 0, fake, fake, fake, fake, fake, fake, 16,
                                        fake, fake, fake, fake, None) == 3
    assert h.rwkv_wkv4_backward_noalloc(1, 16, 64, 0, fake, fake, fake, fake, fake, None, 16,
                                        fake, fake, fake, fake, None) == 1
