"""Guard regions around every output buffer, and the plain-access path of the
WKV-4 kernels.

Each output is carved out of a larger buffer whose head and tail hold a
sentinel; after the call the sentinel must be intact (no write outside the
output) and the output must match the fp64 oracle (the Eagle and Finch backward
too, every one of their six outputs).  compute-sanitizer is not
available, so this is the out-of-bounds check of every entry point.

The WKV-4 calls are exercised on both of their paths: tensors whose bases are
16-byte aligned with C * sizeof(element) a multiple of 16 go through TMA; bases
that are only element aligned (offset by one element) or a C such as 10, 33 or
12 (bf16) take the plain-access instances of the same kernels.  The calls go
through the C ABI with raw pointers."""
import ctypes

import pytest
import torch

import oracle
import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi
from _parity import (TOL_BF16, TOL_Y, assert_close_abs1, assert_close_rms, assert_grads_close, assert_state_close,
                     state_to_ab)

pytestmark = pytest.mark.gpu
GUARD = 64  # elements of sentinel before and after each output (a multiple of 16 bytes for fp32 and bf16)
SENTINEL = 1234567.0  # exact in fp32 and bf16 (1234567 rounds to 1232896 in bf16; compared in the buffer's dtype)


class Guarded:
    """An output tensor of `shape` inside a buffer with GUARD sentinel elements on each side; `offset`
    extra elements shift the output off 16-byte alignment."""

    def __init__(self, shape, dtype, dev, offset=0):
        n = 1
        for s in shape:
            n *= s
        self.n, self.lo = n, GUARD + offset
        self.buf = torch.full((GUARD + offset + n + GUARD,), SENTINEL, dtype=dtype, device=dev)
        self.sentinel = self.buf[0].item()
        self.t = self.buf[self.lo:self.lo + n].view(shape)

    def ptr(self):
        return ctypes.c_void_p(self.t.data_ptr())

    def check(self, what):
        head, tail = self.buf[:self.lo], self.buf[self.lo + self.n:]
        assert torch.all(head == self.sentinel), f"{what}: write before the output"
        assert torch.all(tail == self.sentinel), f"{what}: write after the output"


def _shifted(x, offset):
    """A copy of x whose base is `offset` elements past a 16-byte boundary."""
    buf = torch.empty(x.numel() + 16, dtype=x.dtype, device=x.device)
    t = buf[offset:offset + x.numel()].view(x.shape)
    t.copy_(x)
    return t


CASES = [  # (B, T, C, dtype, offset): the first two go through TMA, the rest take the plain path
    (2, 100, 64, torch.float32, 0),
    (2, 77, 64, torch.bfloat16, 0),
    (3, 77, 33, torch.float32, 0),
    (2, 90, 10, torch.float32, 1),
    (2, 70, 64, torch.float32, 1),
    (2, 85, 12, torch.bfloat16, 1),
    (1, 40, 40, torch.bfloat16, 3),
]


def _ids(c):
    B, T, C, dt, off = c
    return f"{B}x{T}x{C}-{'bf16' if dt == torch.bfloat16 else 'f32'}-off{off}"


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_wkv4_forward_backward_guarded(cuda_device, case):
    B, T, C, dt, off = case
    dev = cuda_device
    bf16 = dt == torch.bfloat16
    p = wi.wkv4_problem(B, T, C, 71, outliers=True, with_gy=True, dtype=dt)
    g = {k: _shifted(v.to(dev), off) if v.dim() == 3 else v.to(dev) for k, v in p.items()}
    h = rw.lib()
    nck = int(h.rwkv_wkv4_num_checkpoints(T, 16))
    y = Guarded((B, T, C), dt, dev, off)
    st = Guarded((3, B, C), torch.float32, dev)
    ck = Guarded((nck, 3, B, C), torch.float32, dev)
    P, S = rw._ptr, rw._stream(None)
    code = rw.BF16 if bf16 else rw.F32
    for algo in (rw.ALGO_SEQUENTIAL, rw.ALGO_CHUNKED):
        wsb = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, algo))
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
        assert h.rwkv_wkv4_forward(B, T, C, code, P(g["w"]), P(g["u"]), P(g["k"]), P(g["v"]), y.ptr(), None,
                                   st.ptr(), ck.ptr(), 16, algo, P(ws), wsb, S) == 0
        rw.rwkv_check_device_error()
        for b_, name in ((y, "y"), (st, "state"), (ck, "checkpoints")):
            b_.check(f"algo {algo} {name}")
        ref, ref_st = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)
        if bf16:
            assert_close_rms(y.t, ref, TOL_BF16, "y bf16")
        else:
            assert_close_abs1(y.t, ref, TOL_Y, "y")
            assert_state_close(st.t, ref_st)
        for j in range(1, nck):
            _, s_j = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :16 * j], p["v"][:, :16 * j], return_state=True)
            if not bf16:
                assert_state_close(ck.t[j], s_j, f"ckpt[{j}]")
    gk, gv = Guarded((B, T, C), dt, dev, off), Guarded((B, T, C), dt, dev, off)
    gw, gu = Guarded((C,), torch.float32, dev), Guarded((C,), torch.float32, dev)
    for use_ckpt in (True, False):
        wsb = int(h.rwkv_wkv4_backward_workspace_bytes(B, T, C, 16, 1 if use_ckpt else 0))
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        assert h.rwkv_wkv4_backward(B, T, C, code, P(g["w"]), P(g["u"]), P(g["k"]), P(g["v"]), P(g["gy"]), None,
                                    ck.ptr() if use_ckpt else None, 16, gk.ptr(), gv.ptr(), gw.ptr(), gu.ptr(),
                                    P(ws), wsb, S) == 0
        rw.rwkv_check_device_error()
        for b_, name in ((gk, "gk"), (gv, "gv"), (gw, "gw"), (gu, "gu")):
            b_.check(name)
        r = oracle.wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["gy"])
        if bf16:
            for got, ref, name in zip((gk.t, gv.t, gw.t, gu.t), r, ("gk", "gv", "gw", "gu")):
                assert_close_rms(got, ref, TOL_BF16, name + " bf16")
        else:
            assert_grads_close((gk.t, gv.t, gw.t, gu.t), r, f"ckpt={use_ckpt} ")


@pytest.mark.parametrize("case", CASES[::2], ids=[_ids(c) for c in CASES[::2]])
def test_wkv4_gated_guarded(cuda_device, case):
    B, T, C, dt, off = case
    dev = cuda_device
    bf16 = dt == torch.bfloat16
    p = wi.wkv4_problem(B, T, C, 72, outliers=True, with_gy=True, gated=True, dtype=dt)
    g = {k: _shifted(v.to(dev), off) if v.dim() == 3 else v.to(dev) for k, v in p.items()}
    h = rw.lib()
    P, S = rw._ptr, rw._stream(None)
    code = rw.BF16 if bf16 else rw.F32
    nck = int(h.rwkv_wkv4_num_checkpoints(T, 16))
    o = Guarded((B, T, C), dt, dev, off)
    ck = Guarded((nck, 3, B, C), torch.float32, dev)
    wsb = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, rw.ALGO_AUTO))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    assert h.rwkv_wkv4_forward_gated(B, T, C, code, P(g["w"]), P(g["u"]), P(g["k"]), P(g["v"]), P(g["r"]), o.ptr(),
                                     None, None, ck.ptr(), 16, rw.ALGO_AUTO, P(ws), wsb, S) == 0
    rw.rwkv_check_device_error()
    o.check("o")
    ck.check("checkpoints")
    ref_o = oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], p["r"])
    if bf16:
        assert_close_rms(o.t, ref_o, TOL_BF16, "o bf16")
    else:
        assert_close_abs1(o.t, ref_o, TOL_Y, "o")
    outs = [Guarded((B, T, C), dt, dev, off) for _ in range(3)] + [Guarded((C,), torch.float32, dev)
                                                                   for _ in range(2)]
    wsb = int(h.rwkv_wkv4_backward_workspace_bytes(B, T, C, 16, 1))
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    assert h.rwkv_wkv4_backward_gated(B, T, C, code, P(g["w"]), P(g["u"]), P(g["k"]), P(g["v"]), P(g["r"]),
                                      P(g["go"]), None, ck.ptr(), 16, *(x.ptr() for x in outs), P(ws), wsb, S) == 0
    rw.rwkv_check_device_error()
    for x, name in zip(outs, ("gk", "gv", "gr", "gw", "gu")):
        x.check(name)
    r = oracle.wkv4_gated_backward(p["w"], p["u"], p["k"], p["v"], p["r"], p["go"])
    if bf16:
        for x, ref, name in zip(outs, r, ("gk", "gv", "gr", "gw", "gu")):
            assert_close_rms(x.t, ref, TOL_BF16, name + " bf16")
    else:
        assert_grads_close(tuple(x.t for x in outs), r, "gated ", names=("gk", "gv", "gr", "gw", "gu"))


@pytest.mark.parametrize("C,dt", [(64, torch.float32), (10, torch.float32), (12, torch.bfloat16)])
def test_wkv4_step_guarded(cuda_device, C, dt):
    B, T = 3, 20
    dev = cuda_device
    p = wi.wkv4_problem(B, T, C, 73, outliers=True, dtype=dt)
    g = {k: v.to(dev) for k, v in p.items()}
    h = rw.lib()
    st = Guarded((3, B, C), torch.float32, dev)
    st.t.zero_()
    ys = []
    for t in range(T):
        y = Guarded((B, C), dt, dev)
        kt, vt = g["k"][:, t].contiguous(), g["v"][:, t].contiguous()
        assert h.rwkv_wkv4_step(B, C, rw.BF16 if dt == torch.bfloat16 else rw.F32, rw._ptr(g["w"]), rw._ptr(g["u"]),
                                rw._ptr(kt), rw._ptr(vt), y.ptr(), st.ptr(), st.ptr(), rw._stream(None)) == 0
        torch.cuda.synchronize()
        y.check(f"y step {t}")
        st.check(f"state step {t}")
        ys.append(y.t.clone())
    ref = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    if dt == torch.bfloat16:
        assert_close_rms(torch.stack(ys, 1), ref, TOL_BF16, "y bf16")
    else:
        assert_close_abs1(torch.stack(ys, 1), ref, TOL_Y, "y")


@pytest.mark.parametrize("finch", [False, True])
def test_matrix_state_guarded(cuda_device, finch):
    B, T, H = 2, 150, 3
    dev = cuda_device
    # one problem of T + 1 tokens: the forward runs over the first T, the decode step takes the last
    q = (wi.wkv6_problem if finch else wi.wkv5_problem)(B, T + 1, H, 64, seed=74)
    names = ("r", "k", "v", "omega") if finch else ("r", "k", "v")
    p = {n: (q[n][:, :T].contiguous() if n in names else q[n]) for n in q}
    g = {k: v.to(dev) for k, v in p.items()}
    h = rw.lib()
    P, S = rw._ptr, rw._stream(None)
    y = Guarded((B, T, H, 64), torch.bfloat16, dev)
    so = Guarded((B, H, 64, 64), torch.float32, dev)
    fwd = h.rwkv_wkv6_forward if finch else h.rwkv_wkv5_forward
    wsb = int((h.rwkv_wkv6_forward_workspace_bytes if finch else h.rwkv_wkv5_forward_workspace_bytes)(B, T, H, 64))
    ws = Guarded((max(wsb, 4) // 4,), torch.float32, dev)  # the scratch, fenced by sentinels too
    assert fwd(B, T, H, 64, P(g["r"]), P(g["k"]), P(g["v"]), P(g["omega"]), P(g["u"]), y.ptr(), None, so.ptr(),
               ws.ptr(), wsb, S) == 0
    rw.rwkv_check_device_error()
    y.check("y")
    so.check("s_out")
    ws.check("workspace")
    ref, ref_s = (oracle.wkv6_forward if finch else oracle.wkv5_forward)(p["r"], p["k"], p["v"], p["omega"], p["u"],
                                                                         return_state=True)
    assert_close_rms(y.t, ref, TOL_BF16, "y")
    assert_close_rms(so.t, ref_s, TOL_BF16, "s_out")
    # one decode step from that state, into guarded outputs
    tok = {n: q[n][:, T].contiguous().to(dev) for n in names}
    ys = Guarded((B, H, 64), torch.bfloat16, dev)
    s1 = Guarded((B, H, 64, 64), torch.float32, dev)
    step = h.rwkv_wkv6_step if finch else h.rwkv_wkv5_step
    om = tok["omega"] if finch else g["omega"]
    assert step(B, H, 64, P(tok["r"]), P(tok["k"]), P(tok["v"]), P(om), P(g["u"]), ys.ptr(), so.ptr(), s1.ptr(),
                S) == 0
    torch.cuda.synchronize()
    ys.check("step y")
    s1.check("step s_out")
    ref1 = (oracle.wkv6_forward if finch else oracle.wkv5_forward)(q["r"], q["k"], q["v"], q["omega"], q["u"])
    assert_close_rms(ys.t, ref1[:, T], TOL_BF16, "step y")


@pytest.mark.parametrize("finch", [False, True])
def test_matrix_state_backward_guarded(cuda_device, finch):
    # the Eagle and Finch backward: every output (gr, gk, gv, gomega, gu, gs_in) carved out of a
    # sentinel-guarded buffer, checked against the oracle
    B, T, H = 2, 130, 3
    dev = cuda_device
    p = (wi.wkv6_problem if finch else wi.wkv5_problem)(B, T, H, 64, seed=75)
    g = wi.wkv5_grads(B, T, H, 64, seed=76, states=True)
    c = {k: v.to(dev) for k, v in list(p.items()) + list(g.items())}
    h = rw.lib()
    P, S = rw._ptr, rw._stream(None)
    outs = {name: Guarded((B, T, H, 64), torch.bfloat16, dev) for name in ("gr", "gk", "gv")}
    outs["gomega"] = Guarded((B, T, H, 64) if finch else (H, 64), torch.float32, dev)
    outs["gu"] = Guarded((H, 64), torch.float32, dev)
    outs["gs_in"] = Guarded((B, H, 64, 64), torch.float32, dev)
    name = "rwkv_wkv6_backward" if finch else "rwkv_wkv5_backward"
    wsb = int(getattr(h, name + "_workspace_bytes")(B, T, H, 64))
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    assert getattr(h, name)(B, T, H, 64, P(c["r"]), P(c["k"]), P(c["v"]), P(c["omega"]), P(c["u"]), P(c["s_in"]),
                            P(c["gy"]), P(c["gs_out"]), outs["gr"].ptr(), outs["gk"].ptr(), outs["gv"].ptr(),
                            outs["gomega"].ptr(), outs["gu"].ptr(), outs["gs_in"].ptr(), P(ws), wsb, S) == 0
    rw.rwkv_check_device_error()
    ref = (oracle.wkv6_backward if finch else oracle.wkv5_backward)(p["r"], p["k"], p["v"], p["omega"], p["u"],
                                                                   g["gy"], s_in=g["s_in"], gs_out=g["gs_out"])
    for key, want in zip(("gr", "gk", "gv", "gomega", "gu", "gs_in"), ref):
        outs[key].check(key)
        assert_close_rms(outs[key].t, want, TOL_BF16, key)


def test_element_misaligned_pointer_is_refused(cuda_device):
    # a float pointer that is not even 4-byte aligned cannot be served by element accesses
    h = rw.lib()
    buf = torch.zeros(4 * 64 * 64 + 4, dtype=torch.float32, device=cuda_device)
    w = torch.ones(64, device=cuda_device)
    bad = ctypes.c_void_p(buf.data_ptr() + 2)
    assert h.rwkv_wkv4_forward(1, 64, 64, rw.F32, rw._ptr(w), rw._ptr(w), bad, bad, bad, None, None, None, 16,
                               rw.ALGO_SEQUENTIAL, None, 0, rw._stream(None)) == 2
