"""Host-side checks of the C-ABI library, no GPU needed: it loads, it exports
every function that include/rwkv_wkv.h declares, and argument validation
answers before any CUDA work is enqueued."""
import ctypes
import os
import re

import pytest

import rwkv_wkv_recurrence_b200 as rw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names += re.findall(r"^RWKV_API\s+[\w\s\*]+?\**\s*(\w+)\s*\(", src, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert "rwkv_wkv4_forward" in names and "rwkv_wkv5_forward" in names and "rwkv_wkv6_forward" in names
    h = ctypes.CDLL(rw.LIB_PATH)
    missing = [n for n in names if not hasattr(h, n)]
    assert not missing, missing


def test_status_strings_and_version():
    h = rw.lib()
    assert h.rwkv_status_string(0) == b"ok"
    for s in range(1, 6):
        assert h.rwkv_status_string(s) not in (b"ok", b"unknown status")
    assert h.rwkv_status_string(99) == b"unknown status"
    assert h.rwkv_version() >> 16 == 1


def test_checkpoint_and_workspace_queries():
    h = rw.lib()
    assert h.rwkv_wkv4_num_checkpoints(4096, 16) == 256
    assert h.rwkv_wkv4_num_checkpoints(4097, 16) == 257
    assert h.rwkv_wkv4_num_checkpoints(0, 16) == 0
    assert h.rwkv_wkv4_num_checkpoints(100, 12) == -1
    assert h.rwkv_wkv4_num_checkpoints(100, 0) == -1
    B, T, C = 8, 4096, 2048
    assert h.rwkv_wkv4_backward_workspace_bytes(B, T, C, 16, 1) == 2 * B * C * 8
    assert h.rwkv_wkv4_backward_workspace_bytes(B, T, C, 16, 0) == 2 * B * C * 8 + 256 * 3 * B * C * 4
    # many channels: the sequential schedule needs no workspace
    assert h.rwkv_wkv4_forward_workspace_bytes(B, T, C, rw.ALGO_AUTO) == 0
    assert h.rwkv_wkv4_forward_workspace_bytes(B, T, C, rw.ALGO_SEQUENTIAL) == 0
    # 192 channel tiles (8 x 768): AUTO keeps the sequential schedule, which measured faster there;
    # 24 tiles (1 x 768) over 4096 steps: AUTO cuts time into segments, one state per segment
    assert h.rwkv_wkv4_forward_workspace_bytes(8, 1024, 768, rw.ALGO_AUTO) == 0
    # (22 segments of 192 steps: per segment and lane a summary as three doubles, and a flag per
    # segment and CTA, for the one-launch form)
    ws = h.rwkv_wkv4_forward_workspace_bytes(1, 4096, 768, rw.ALGO_AUTO)
    assert ws >= 22 * 768 * 3 * 8 + 22 * 24 * 4 and ws < 22 * 768 * 3 * 8 + 4096
    assert h.rwkv_wkv4_forward_workspace_bytes(8, 1024, 768, rw.ALGO_CHUNKED) > 0
    assert h.rwkv_wkv4_forward_workspace_bytes(0, 10, 10, 0) == 0
    # Eagle forward: the heads' 64-token chunks are dealt out to 296 CTAs (two per SM); per CTA
    # a 64 x 64 fp32 summary and a flag, and a ticket counter
    for shape in [(4, 4096, 40), (1, 4096, 40), (8, 4096, 40)]:
        ws = h.rwkv_wkv5_forward_workspace_bytes(*shape, 64)
        assert ws >= 296 * 64 * 64 * 4 + 297 * 4 and ws < 296 * 64 * 64 * 4 + 4096, shape
    ws = h.rwkv_wkv5_forward_workspace_bytes(1, 128, 1, 64)  # two chunks: two CTAs
    assert ws >= 2 * 64 * 64 * 4 + 3 * 4 and ws < 2 * 64 * 64 * 4 + 1024
    assert h.rwkv_wkv5_forward_workspace_bytes(4, 64, 40, 64) == 0  # one chunk per head: one CTA per head
    assert h.rwkv_wkv5_forward_workspace_bytes(4, 4096, 40, 32) == 0
    assert h.rwkv_wkv6_forward_workspace_bytes(4, 4096, 40, 64) == 0  # Finch: one CTA per head


def test_validation_before_any_cuda_work():
    h = rw.lib()
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: every call below fails validation first
    # negative sizes
    assert h.rwkv_wkv4_forward(-1, 4, 4, 0, fake, fake, fake, fake, fake, None, None, None, 16, 0, None, 0,
                               None) == 1
    # bad dtype / algo
    assert h.rwkv_wkv4_forward(1, 4, 4, 7, fake, fake, fake, fake, fake, None, None, None, 16, 0, None, 0,
                               None) == 1
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, None, None, 16, 9, None, 0,
                               None) == 1
    # checkpoint interval not a multiple of 16 / not supported
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, None, fake, 12, 0, None, 0,
                               None) == 1
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, None, fake, 32, 0, None, 0,
                               None) == 2
    # empty problems are a no-op
    assert h.rwkv_wkv4_forward(0, 4, 4, 0, fake, fake, fake, fake, fake, None, None, None, 16, 0, None, 0,
                               None) == 0
    # null required pointers
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, None, fake, fake, fake, fake, None, None, None, 16, 0, None, 0,
                               None) == 1
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, fake, fake, None, fake, fake, None, None, None, 16, 0, None, 0,
                               None) == 1
    # a pointer not aligned to its element (a 16-byte misalignment alone is served by the plain path)
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, fake, fake, P(0x1002), fake, fake, None, None, None, 16, 0, None,
                               0, None) == 2
    assert h.rwkv_wkv4_forward(1, 4, 4, 0, fake, fake, fake, fake, P(0x1001), None, None, None, 16, 0, None,
                               0, None) == 2
    assert h.rwkv_wkv4_forward(1, 4, 4, 1, fake, fake, fake, P(0x1001), fake, None, None, None, 16, 0, None,
                               0, None) == 2
    # chunked schedule without its workspace
    assert h.rwkv_wkv4_forward(8, 1024, 768, 0, fake, fake, fake, fake, fake, None, None, None, 16,
                               rw.ALGO_CHUNKED, None, 0, None) == 3
    assert h.rwkv_wkv4_forward(1, 4096, 768, 0, fake, fake, fake, fake, fake, None, None, None, 16, rw.ALGO_AUTO,
                               None, 0, None) == 3
    # backward: bad interval, missing workspace, null gradient
    assert h.rwkv_wkv4_backward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, fake, 8, fake, fake, fake,
                                fake, fake, 1 << 20, None) == 1
    assert h.rwkv_wkv4_backward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, fake, 16, fake, fake, fake,
                                fake, None, 0, None) == 3
    assert h.rwkv_wkv4_backward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, fake, 16, None, fake, fake,
                                fake, fake, 1 << 20, None) == 1
    # backward: gk or gv not aligned to its element
    assert h.rwkv_wkv4_backward(1, 4, 4, 0, fake, fake, fake, fake, fake, None, fake, 16, P(0x1002), fake,
                                fake, fake, fake, 1 << 20, None) == 2
    assert h.rwkv_wkv4_backward(1, 4, 4, 1, fake, fake, fake, fake, fake, None, fake, 16, fake, P(0x1003),
                                fake, fake, fake, 1 << 20, None) == 2
    # step: null output state
    assert h.rwkv_wkv4_step(2, 4, 0, fake, fake, fake, fake, fake, None, None, None) == 1
    assert h.rwkv_wkv4_step(-2, 4, 0, fake, fake, fake, fake, fake, None, fake, None) == 1
    # WKV-5: only N = 64
    assert h.rwkv_wkv5_forward(1, 4, 2, 32, fake, fake, fake, fake, fake, fake, None, None, None, 0,
                               None) == 2
    assert h.rwkv_wkv5_forward(1, 4, 2, 64, fake, fake, fake, None, fake, fake, None, None, None, 0,
                               None) == 1
    # the slot plan with a workspace that is not 16-byte aligned
    need = h.rwkv_wkv5_forward_workspace_bytes(4, 4096, 40, 64)
    assert h.rwkv_wkv5_forward(4, 4096, 40, 64, fake, fake, fake, fake, fake, fake, None, None, P(0x1004),
                               need, None) == 2
    # the slot plan without the workspace it needs
    assert h.rwkv_wkv5_forward(4, 4096, 40, 64, fake, fake, fake, fake, fake, fake, None, None, None, 0,
                               None) == 3
    assert h.rwkv_wkv5_forward(4, 4096, 40, 64, fake, fake, fake, fake, fake, fake, None, None, fake,
                               h.rwkv_wkv5_forward_workspace_bytes(4, 4096, 40, 64) - 1, None) == 3
    # WKV-5 decode step: only N = 64, output state required, 16-byte aligned states
    assert h.rwkv_wkv5_step(2, 3, 32, fake, fake, fake, fake, fake, fake, None, fake, None) == 2
    assert h.rwkv_wkv5_step(2, 3, 64, fake, fake, fake, fake, fake, fake, None, None, None) == 1
    assert h.rwkv_wkv5_step(2, 3, 64, fake, None, fake, fake, fake, fake, None, fake, None) == 1
    assert h.rwkv_wkv5_step(2, 3, 64, fake, fake, fake, fake, fake, fake, None, P(0x1004), None) == 2
    assert h.rwkv_wkv5_step(2, 3, 64, fake, fake, fake, fake, fake, fake, P(0x1008), fake, None) == 2
    assert h.rwkv_wkv5_step(-2, 3, 64, fake, fake, fake, fake, fake, fake, None, fake, None) == 1
    assert h.rwkv_wkv5_step(0, 3, 64, fake, fake, fake, fake, fake, fake, None, fake, None) == 0
    # gated WKV-4: r and o required and aligned; the backward needs r, go and gr together
    assert h.rwkv_wkv4_forward_gated(1, 4, 4, 0, fake, fake, fake, fake, None, fake, None, None, None, 16, 0,
                                     None, 0, None) == 1
    assert h.rwkv_wkv4_forward_gated(1, 4, 4, 0, fake, fake, fake, fake, fake, None, None, None, None, 16, 0,
                                     None, 0, None) == 1
    assert h.rwkv_wkv4_forward_gated(1, 4, 4, 0, fake, fake, fake, fake, P(0x1002), fake, None, None, None, 16,
                                     0, None, 0, None) == 2
    assert h.rwkv_wkv4_forward_gated(-1, 4, 4, 0, fake, fake, fake, fake, fake, fake, None, None, None, 16, 0,
                                     None, 0, None) == 1
    assert h.rwkv_wkv4_forward_gated(0, 4, 4, 0, fake, fake, fake, fake, fake, fake, None, None, None, 16, 0,
                                     None, 0, None) == 0
    assert h.rwkv_wkv4_backward_gated(1, 4, 4, 0, fake, fake, fake, fake, None, fake, None, fake, 16, fake,
                                      fake, fake, fake, fake, fake, 1 << 20, None) == 1
    assert h.rwkv_wkv4_backward_gated(1, 4, 4, 0, fake, fake, fake, fake, fake, fake, None, fake, 16, fake,
                                      fake, None, fake, fake, fake, 1 << 20, None) == 1
    assert h.rwkv_wkv4_backward_gated(1, 4, 4, 0, fake, fake, fake, fake, None, None, None, fake, 16, fake,
                                      fake, None, fake, fake, fake, 1 << 20, None) == 1
    assert h.rwkv_wkv4_backward_gated(1, 4, 4, 0, fake, fake, fake, fake, fake, fake, None, fake, 16, fake,
                                      fake, P(0x1002), fake, fake, fake, 1 << 20, None) == 2
    assert h.rwkv_wkv4_backward_gated(1, 4, 4, 0, fake, fake, fake, fake, fake, fake, None, fake, 16, fake,
                                      fake, fake, fake, fake, None, 0, None) == 3
    # WKV-6 forward: only N = 64; omega required and 16-byte aligned (TMA); T = 0 without s_out is a no-op
    assert h.rwkv_wkv6_forward(1, 4, 2, 32, fake, fake, fake, fake, fake, fake, None, None, None, 0, None) == 2
    assert h.rwkv_wkv6_forward(1, 4, 2, 64, fake, fake, fake, None, fake, fake, None, None, None, 0, None) == 1
    assert h.rwkv_wkv6_forward(1, 4, 2, 64, fake, fake, fake, fake, None, fake, None, None, None, 0, None) == 1
    assert h.rwkv_wkv6_forward(1, 4, 2, 64, fake, fake, fake, fake, fake, None, None, None, None, 0, None) == 1
    assert h.rwkv_wkv6_forward(1, 4, 2, 64, fake, fake, fake, P(0x1004), fake, fake, None, None, None, 0,
                               None) == 2
    assert h.rwkv_wkv6_forward(1, 4, 2, 64, fake, fake, fake, fake, fake, P(0x1008), None, None, None, 0,
                               None) == 2
    assert h.rwkv_wkv6_forward(-1, 4, 2, 64, fake, fake, fake, fake, fake, fake, None, None, None, 0, None) == 1
    assert h.rwkv_wkv6_forward(0, 4, 2, 64, fake, fake, fake, fake, fake, fake, None, None, None, 0, None) == 0
    assert h.rwkv_wkv6_forward(1, 0, 2, 64, None, None, None, None, fake, None, None, None, None, 0, None) == 0
    # WKV-6 decode step: as the WKV-5 step, with a per-stream omega
    assert h.rwkv_wkv6_step(2, 3, 32, fake, fake, fake, fake, fake, fake, None, fake, None) == 2
    assert h.rwkv_wkv6_step(2, 3, 64, fake, fake, fake, None, fake, fake, None, fake, None) == 1
    assert h.rwkv_wkv6_step(2, 3, 64, fake, fake, fake, fake, fake, fake, None, None, None) == 1
    assert h.rwkv_wkv6_step(2, 3, 64, fake, fake, fake, fake, fake, fake, None, P(0x1004), None) == 2
    assert h.rwkv_wkv6_step(0, 3, 64, fake, fake, fake, fake, fake, fake, None, fake, None) == 0
    # WKV-5 / WKV-6 backward: only N = 64; the tensors and gradients required and 16-byte aligned; the
    # workspace at least the query's size; B = 0 a no-op
    for name in ("rwkv_wkv5_backward", "rwkv_wkv6_backward"):
        f = getattr(h, name)
        ok = [fake] * 15  # r, k, v, omega, u, s_in, gy, gs_out, gr, gk, gv, gomega, gu, gs_in, workspace

        def call(B=1, T=4, H=2, N=64, ptrs=None, wsb=1 << 30):
            a = list(ok if ptrs is None else ptrs)
            return f(B, T, H, N, *a[:14], a[14], wsb, None)

        def with_ptr(i, val):
            a = list(ok)
            a[i] = val
            return a

        assert call(N=32) == 2, name
        assert call(B=-1) == 1, name
        assert call(B=0) == 0, name
        assert call(ptrs=with_ptr(0, None)) == 1, name    # r
        assert call(ptrs=with_ptr(6, None)) == 1, name    # gy
        assert call(ptrs=with_ptr(12, None)) == 1, name   # gu
        assert call(ptrs=with_ptr(10, None)) == 1, name   # gv
        assert call(ptrs=with_ptr(1, P(0x1008))) == 2, name
        assert call(ptrs=with_ptr(8, P(0x1004))) == 2, name
        assert call(ptrs=with_ptr(14, None)) == 3, name   # no workspace
        need = int(getattr(h, name + "_workspace_bytes")(1, 4, 2, 64))
        assert need > 0 and call(wsb=need - 1) == 3, name
    # the Finch backward runs one CTA per 64-token chunk: more than 2^31 - 1 chunks is refused
    big = h.rwkv_wkv6_backward(1 << 16, 1 << 17, 1 << 10, 64, *([fake] * 15), 1 << 62, None)
    assert big == 2


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(rw, "_lib", None)
    monkeypatch.setattr(rw, "LIB_PATH", "/nonexistent/librwkv_wkv.so")
    with pytest.raises(RuntimeError, match="missing"):
        rw.lib()
