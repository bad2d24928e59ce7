"""The failure path of the kernels' bounded waits, on the GPU, without a fault
or a hang: the test hook makes every CTA's load-issuing thread arm its barrier
and issue no load, with a short wait limit, so the first wait of each CTA runs
out with nothing in flight.  The kernel records RWKV_ERR_DEVICE_TIMEOUT and its
CTAs leave; rwkv_check_device_error reports it once and clears it; with the hook
off the same context computes correct results again."""
import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import TOL_BF16, TOL_Y, assert_close_abs1, assert_close_rms

pytestmark = pytest.mark.gpu
TIMEOUT = 5  # RWKV_ERR_DEVICE_TIMEOUT
LIMIT_NS = 20_000_000  # 20 ms


def _calls(dev):
    p = {k: v.to(dev) for k, v in wi.wkv4_problem(2, 130, 64, 61, outliers=True, with_gy=True).items()}
    e = {k: v.to(dev) for k, v in wi.wkv5_problem(1, 70, 2, 64, seed=62).items()}
    f = {k: v.to(dev) for k, v in wi.wkv6_problem(1, 70, 2, 64, seed=63).items()}
    # 160 heads of 4 chunks over 296 CTAs that wait for one another's summaries
    c = {k: v.to(dev) for k, v in wi.wkv5_problem(4, 200, 40, 64, seed=64).items()}
    ck = rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"], p["v"], checkpoints=True)[1]
    torch.cuda.synchronize()
    return {
        "wkv4 forward": lambda: rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"], p["v"], algo=rw.ALGO_SEQUENTIAL),
        "wkv4 chunked forward": lambda: rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"], p["v"], algo=rw.ALGO_CHUNKED),
        "wkv4 backward": lambda: rw.rwkv_wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["gy"], ckpt=ck),
        "eagle forward": lambda: rw.rwkv_wkv5_forward(e["r"], e["k"], e["v"], e["omega"], e["u"]),
        "eagle forward, split heads": lambda: rw.rwkv_wkv5_forward(c["r"], c["k"], c["v"], c["omega"], c["u"]),
        "finch forward": lambda: rw.rwkv_wkv6_forward(f["r"], f["k"], f["v"], f["omega"], f["u"]),
    }


def test_bounded_waits_give_up_and_report_a_timeout(cuda_device):
    h = rw.lib()
    calls = _calls(cuda_device)
    assert h.rwkv_check_device_error(rw._stream(None)) == 0
    assert h.rwkv_debug_set_wait_limit_ns(LIMIT_NS) == 0
    assert h.rwkv_debug_withhold_loads(1) == 0
    try:
        for name, call in calls.items():
            call()  # enqueues normally; the kernel's waits give up on the device
            assert h.rwkv_check_device_error(rw._stream(None)) == TIMEOUT, name
            assert h.rwkv_check_device_error(rw._stream(None)) == 0, name + ": the word was not cleared"
    finally:
        assert h.rwkv_debug_withhold_loads(0) == 0
        assert h.rwkv_debug_set_wait_limit_ns(0) == 0
    # the same context works again: every call completes without a timeout and matches the oracle
    for name, call in calls.items():
        call()
        assert h.rwkv_check_device_error(rw._stream(None)) == 0, name
    p = wi.wkv4_problem(2, 130, 64, 61, outliers=True)
    assert_close_abs1(calls["wkv4 forward"](), oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"]), TOL_Y, "y")
    q = wi.wkv5_problem(1, 70, 2, 64, seed=62)
    assert_close_rms(calls["eagle forward"](), oracle.wkv5_forward(q["r"], q["k"], q["v"], q["omega"], q["u"]),
                     TOL_BF16, "eagle y")
