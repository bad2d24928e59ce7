"""Python binding of the B200 WKV operator library (``librwkv_wkv.so``).

Two layers, both argument marshalling only (every step of the operator runs in
the library's CUDA kernels):

* ``lib()`` returns the ctypes handle whose functions carry the exact C-ABI
  names and signatures of ``include/rwkv_wkv.h`` (``rwkv_wkv4_forward``,
  ``rwkv_wkv4_backward``, ``rwkv_wkv4_step``, ``rwkv_wkv5_forward``, ...).
* ``rwkv_wkv4_forward`` & co. below take torch CUDA tensors, allocate outputs
  and workspace with torch, pass raw device pointers and the current torch
  stream to the C call, and raise ``RwkvError`` on a non-OK status.

There is no fallback: if the library is missing or a call fails, this raises.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "LIB_PATH", "lib", "RwkvError", "RWKV_OK", "F32", "BF16", "ALGO_AUTO", "ALGO_SEQUENTIAL",
    "ALGO_CHUNKED", "CHUNK_LEN", "NOALLOC_MAX_LANES", "rwkv_wkv4_forward", "rwkv_wkv4_backward",
    "rwkv_wkv4_backward_noalloc", "rwkv_wkv4_step", "rwkv_wkv4_forward_gated", "rwkv_wkv4_backward_gated",
    "rwkv_wkv5_forward", "rwkv_wkv5_backward", "rwkv_wkv5_step", "rwkv_wkv6_forward", "rwkv_wkv6_backward",
    "rwkv_wkv6_step", "rwkv_check_device_error",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librwkv_wkv.so")

RWKV_OK = 0
F32, BF16 = 0, 1
ALGO_AUTO, ALGO_SEQUENTIAL, ALGO_CHUNKED = 0, 1, 2
CHUNK_LEN = 16  # checkpoint interval of the WKV-4 forward/backward pair
NOALLOC_MAX_LANES = 262144  # RWKV_NOALLOC_MAX_LANES: largest B*C of rwkv_wkv4_backward_noalloc

_lib = None


class RwkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib().rwkv_status_string(status).decode()
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


def lib():
    """ctypes handle of librwkv_wkv.so with argtypes set from the C header."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m rwkv_wkv_recurrence_b200._build` (needs nvcc)")
    h = ctypes.CDLL(LIB_PATH)
    I64, P, S, I = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    sig = {
        "rwkv_status_string": ([I], ctypes.c_char_p),
        "rwkv_version": ([], I),
        "rwkv_wkv4_num_checkpoints": ([I64, I64], I64),
        "rwkv_wkv4_forward_workspace_bytes": ([I64, I64, I64, I], S),
        "rwkv_wkv4_forward": ([I64, I64, I64, I, P, P, P, P, P, P, P, P, I64, I, P, S, P], I),
        "rwkv_wkv4_backward_workspace_bytes": ([I64, I64, I64, I64, I], S),
        "rwkv_wkv4_backward": ([I64, I64, I64, I, P, P, P, P, P, P, P, I64, P, P, P, P, P, S, P], I),
        "rwkv_wkv4_step": ([I64, I64, I, P, P, P, P, P, P, P, P], I),
        "rwkv_wkv4_forward_gated": ([I64, I64, I64, I, P, P, P, P, P, P, P, P, P, I64, I, P, S, P], I),
        "rwkv_wkv4_backward_gated": ([I64, I64, I64, I, P, P, P, P, P, P, P, P, I64, P, P, P, P, P, P, S, P], I),
        "rwkv_wkv5_forward_workspace_bytes": ([I64, I64, I64, I64], S),
        "rwkv_wkv5_forward": ([I64, I64, I64, I64, P, P, P, P, P, P, P, P, P, S, P], I),
        "rwkv_wkv4_backward_noalloc": ([I64, I64, I64, I, P, P, P, P, P, P, I64, P, P, P, P, P], I),
        "rwkv_wkv5_step": ([I64, I64, I64, P, P, P, P, P, P, P, P, P], I),
        "rwkv_wkv5_backward_workspace_bytes": ([I64, I64, I64, I64], S),
        "rwkv_wkv5_backward": ([I64, I64, I64, I64] + [P] * 15 + [S, P], I),
        "rwkv_wkv6_forward_workspace_bytes": ([I64, I64, I64, I64], S),
        "rwkv_wkv6_forward": ([I64, I64, I64, I64, P, P, P, P, P, P, P, P, P, S, P], I),
        "rwkv_wkv6_backward_workspace_bytes": ([I64, I64, I64, I64], S),
        "rwkv_wkv6_backward": ([I64, I64, I64, I64] + [P] * 15 + [S, P], I),
        "rwkv_wkv6_step": ([I64, I64, I64, P, P, P, P, P, P, P, P, P], I),
        "rwkv_check_device_error": ([P], I),
        "rwkv_debug_set_wait_limit_ns": ([ctypes.c_uint64], I),
        "rwkv_debug_withhold_loads": ([I], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(h, name)
        f.argtypes = args
        f.restype = res
    _lib = h
    return h


# ------------------------------------------------------------------ helpers
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != RWKV_OK:
        raise RwkvError(fn, status)


def _dtype_code(t):
    import torch

    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"WKV-4 tensors must be float32 or bfloat16, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("WKV tensors must be CUDA tensors (use .cuda())")
            if not t.is_contiguous():
                raise ValueError("WKV tensors must be contiguous")


def _f32(name, t, n):
    import torch

    if t.dtype != torch.float32 or t.numel() != n:
        raise ValueError(f"{name} must be float32 with {n} elements")


# ------------------------------------------------------------------ WKV-4
def rwkv_wkv4_forward(w, u, k, v, state_in=None, *, return_state=False, checkpoints=False,
                      algo=ALGO_AUTO, stream=None, out=None):
    """WKV-4 forward.  k, v [B,T,C] (fp32 or bf16); w, u [C] fp32.

    Returns y, plus the final state [3,B,C] if ``return_state`` and the
    checkpoints [ceil(T/16),3,B,C] for ``rwkv_wkv4_backward`` if ``checkpoints``.
    """
    import torch

    _need_cuda(w, u, k, v, state_in)
    B, T, C = k.shape
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k and v must have the same shape and dtype")
    _f32("w", w, C)
    _f32("u", u, C)
    if state_in is not None:
        _f32("state_in", state_in, 3 * B * C)
    h = lib()
    y = torch.empty_like(k) if out is None else out
    st = torch.empty((3, B, C), dtype=torch.float32, device=k.device) if return_state else None
    nck = int(h.rwkv_wkv4_num_checkpoints(T, CHUNK_LEN))
    ck = torch.empty((nck, 3, B, C), dtype=torch.float32, device=k.device) if checkpoints else None
    wsb = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, algo))
    ws = torch.empty(wsb, dtype=torch.uint8, device=k.device) if wsb else None
    _check("rwkv_wkv4_forward",
           h.rwkv_wkv4_forward(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y),
                               _ptr(state_in), _ptr(st), _ptr(ck), CHUNK_LEN, algo, _ptr(ws), wsb,
                               _stream(stream)))
    res = (y,)
    if return_state:
        res += (st,)
    if checkpoints:
        res += (ck,)
    return res[0] if len(res) == 1 else res


def rwkv_wkv4_backward(w, u, k, v, gy, ckpt=None, state_in=None, *, stream=None, out=None):
    """WKV-4 backward: returns (gk, gv, gw, gu) for L = sum(gy * y).

    ``ckpt`` are the forward's checkpoints (or None to recompute them)."""
    import torch

    _need_cuda(w, u, k, v, gy, ckpt, state_in)
    B, T, C = k.shape
    for name, t in (("v", v), ("gy", gy)):
        if t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError(f"{name} must match k in shape and dtype")
    _f32("w", w, C)
    _f32("u", u, C)
    h = lib()
    if ckpt is not None:
        _f32("ckpt", ckpt, int(h.rwkv_wkv4_num_checkpoints(T, CHUNK_LEN)) * 3 * B * C)
    if state_in is not None:
        _f32("state_in", state_in, 3 * B * C)
    if out is None:
        gk, gv = torch.empty_like(k), torch.empty_like(v)
        gw = torch.empty(C, dtype=torch.float32, device=k.device)
        gu = torch.empty(C, dtype=torch.float32, device=k.device)
    else:
        gk, gv, gw, gu = out
    wsb = int(h.rwkv_wkv4_backward_workspace_bytes(B, T, C, CHUNK_LEN, 1 if ckpt is not None else 0))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=k.device)
    _check("rwkv_wkv4_backward",
           h.rwkv_wkv4_backward(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(gy),
                                _ptr(state_in), _ptr(ckpt), CHUNK_LEN, _ptr(gk), _ptr(gv), _ptr(gw),
                                _ptr(gu), _ptr(ws), wsb, _stream(stream)))
    return gk, gv, gw, gu


def rwkv_wkv4_forward_gated(w, u, k, v, r, state_in=None, *, return_state=False, checkpoints=False,
                            algo=ALGO_AUTO, stream=None, out=None):
    """Receptance-gated WKV-4 forward: o = sigmoid(r) * WKV in one pass.  k, v, r
    [B,T,C] (fp32 or bf16); w, u [C] fp32.  Returns o (plus the state and the
    checkpoints as ``rwkv_wkv4_forward``)."""
    import torch

    _need_cuda(w, u, k, v, r, state_in)
    B, T, C = k.shape
    for name, t in (("v", v), ("r", r)):
        if t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError(f"{name} must match k in shape and dtype")
    _f32("w", w, C)
    _f32("u", u, C)
    if state_in is not None:
        _f32("state_in", state_in, 3 * B * C)
    h = lib()
    o = torch.empty_like(k) if out is None else out
    st = torch.empty((3, B, C), dtype=torch.float32, device=k.device) if return_state else None
    nck = int(h.rwkv_wkv4_num_checkpoints(T, CHUNK_LEN))
    ck = torch.empty((nck, 3, B, C), dtype=torch.float32, device=k.device) if checkpoints else None
    wsb = int(h.rwkv_wkv4_forward_workspace_bytes(B, T, C, algo))
    ws = torch.empty(wsb, dtype=torch.uint8, device=k.device) if wsb else None
    _check("rwkv_wkv4_forward_gated",
           h.rwkv_wkv4_forward_gated(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(o),
                                     _ptr(state_in), _ptr(st), _ptr(ck), CHUNK_LEN, algo, _ptr(ws), wsb,
                                     _stream(stream)))
    res = (o,)
    if return_state:
        res += (st,)
    if checkpoints:
        res += (ck,)
    return res[0] if len(res) == 1 else res


def rwkv_wkv4_backward_gated(w, u, k, v, r, go, ckpt=None, state_in=None, *, stream=None, out=None):
    """Backward of the gated forward: returns (gk, gv, gr, gw, gu) for
    L = sum(go * o), o = sigmoid(r) * WKV."""
    import torch

    _need_cuda(w, u, k, v, r, go, ckpt, state_in)
    B, T, C = k.shape
    for name, t in (("v", v), ("r", r), ("go", go)):
        if t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError(f"{name} must match k in shape and dtype")
    _f32("w", w, C)
    _f32("u", u, C)
    h = lib()
    if ckpt is not None:
        _f32("ckpt", ckpt, int(h.rwkv_wkv4_num_checkpoints(T, CHUNK_LEN)) * 3 * B * C)
    if state_in is not None:
        _f32("state_in", state_in, 3 * B * C)
    if out is None:
        gk, gv, gr = torch.empty_like(k), torch.empty_like(v), torch.empty_like(r)
        gw = torch.empty(C, dtype=torch.float32, device=k.device)
        gu = torch.empty(C, dtype=torch.float32, device=k.device)
    else:
        gk, gv, gr, gw, gu = out
    wsb = int(h.rwkv_wkv4_backward_workspace_bytes(B, T, C, CHUNK_LEN, 1 if ckpt is not None else 0))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=k.device)
    _check("rwkv_wkv4_backward_gated",
           h.rwkv_wkv4_backward_gated(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                      _ptr(go), _ptr(state_in), _ptr(ckpt), CHUNK_LEN, _ptr(gk), _ptr(gv),
                                      _ptr(gr), _ptr(gw), _ptr(gu), _ptr(ws), wsb, _stream(stream)))
    return gk, gv, gr, gw, gu


def rwkv_wkv4_backward_noalloc(w, u, k, v, gy, ckpt, *, stream=None, out=None):
    """WKV-4 backward through the entry point that allocates no device memory
    and takes no workspace (its scratch is a fixed array inside the library,
    shared by all calls; see include/rwkv_wkv.h).  ``ckpt`` is required.
    Output tensors are still the caller's: pass ``out=(gk, gv, gw, gu)`` to
    keep this call free of allocations from Python too."""
    import torch

    _need_cuda(w, u, k, v, gy, ckpt)
    B, T, C = k.shape
    for name, t in (("v", v), ("gy", gy)):
        if t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError(f"{name} must match k in shape and dtype")
    _f32("w", w, C)
    _f32("u", u, C)
    _f32("ckpt", ckpt, int(lib().rwkv_wkv4_num_checkpoints(T, CHUNK_LEN)) * 3 * B * C)
    if out is None:
        gk, gv = torch.empty_like(k), torch.empty_like(v)
        gw = torch.empty(C, dtype=torch.float32, device=k.device)
        gu = torch.empty(C, dtype=torch.float32, device=k.device)
    else:
        gk, gv, gw, gu = out
    _check("rwkv_wkv4_backward_noalloc",
           lib().rwkv_wkv4_backward_noalloc(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(gy),
                                            _ptr(ckpt), CHUNK_LEN, _ptr(gk), _ptr(gv), _ptr(gw), _ptr(gu),
                                            _stream(stream)))
    return gk, gv, gw, gu


def rwkv_wkv4_step(w, u, k, v, state, *, state_out=None, stream=None, out=None):
    """One decode token: k, v [B,C]; state [3,B,C] updated in place unless
    ``state_out`` is given.  Returns y [B,C]."""
    import torch

    _need_cuda(w, u, k, v, state, state_out)
    B, C = k.shape
    y = torch.empty_like(k) if out is None else out
    so = state if state_out is None else state_out
    _check("rwkv_wkv4_step",
           lib().rwkv_wkv4_step(B, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y),
                                _ptr(state), _ptr(so), _stream(stream)))
    return y


# ------------------------------------------------------------------ WKV-5
def rwkv_wkv5_forward(r, k, v, omega, u, s_in=None, *, return_state=False, stream=None, out=None):
    """Eagle / RWKV-5 forward: r, k, v [B,T,H,N] bf16; omega, u [H,N] fp32."""
    import torch

    _need_cuda(r, k, v, omega, u, s_in)
    B, T, H, N = r.shape
    for t in (r, k, v):
        if t.dtype != torch.bfloat16 or t.shape != r.shape:
            raise ValueError("r, k, v must be bf16 of the same shape")
    _f32("omega", omega, H * N)
    _f32("u", u, H * N)
    h = lib()
    y = torch.empty_like(r) if out is None else out
    so = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device) if return_state else None
    wsb = int(h.rwkv_wkv5_forward_workspace_bytes(B, T, H, N))
    ws = torch.empty(wsb, dtype=torch.uint8, device=r.device) if wsb else None
    _check("rwkv_wkv5_forward",
           h.rwkv_wkv5_forward(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(y),
                               _ptr(s_in), _ptr(so), _ptr(ws), wsb, _stream(stream)))
    return (y, so) if return_state else y


def rwkv_wkv5_backward(r, k, v, omega, u, gy, s_in=None, gs_out=None, *, want_gs_in=False, stream=None):
    """Eagle / RWKV-5 backward: gradients of sum(gy * y) + sum(gs_out * s_out).  r, k, v, gy
    [B,T,H,N] bf16; omega, u [H,N] fp32; s_in, gs_out [B,H,N,N] fp32 or None.  Returns
    (gr, gk, gv, gomega, gu) and, with ``want_gs_in``, the gradient of s_in as well."""
    import torch

    _need_cuda(r, k, v, omega, u, gy, s_in, gs_out)
    B, T, H, N = r.shape
    for t in (r, k, v, gy):
        if t.dtype != torch.bfloat16 or t.shape != r.shape:
            raise ValueError("r, k, v, gy must be bf16 of the same shape")
    _f32("omega", omega, H * N)
    _f32("u", u, H * N)
    for name, t in (("s_in", s_in), ("gs_out", gs_out)):
        if t is not None:
            _f32(name, t, B * H * N * N)
    h = lib()
    gr, gk, gv = torch.empty_like(r), torch.empty_like(k), torch.empty_like(v)
    gomega = torch.empty((H, N), dtype=torch.float32, device=r.device)
    gu = torch.empty((H, N), dtype=torch.float32, device=r.device)
    gsi = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device) if want_gs_in else None
    wsb = int(h.rwkv_wkv5_backward_workspace_bytes(B, T, H, N))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=r.device)
    _check("rwkv_wkv5_backward",
           h.rwkv_wkv5_backward(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(s_in), _ptr(gy),
                                _ptr(gs_out), _ptr(gr), _ptr(gk), _ptr(gv), _ptr(gomega), _ptr(gu), _ptr(gsi),
                                _ptr(ws), wsb, _stream(stream)))
    res = (gr, gk, gv, gomega, gu)
    return res + (gsi,) if want_gs_in else res


def rwkv_wkv6_backward(r, k, v, omega, u, gy, s_in=None, gs_out=None, *, want_gs_in=False, stream=None):
    """Finch / RWKV-6 backward: gradients of sum(gy * y) + sum(gs_out * s_out).  r, k, v, gy
    [B,T,H,N] bf16; omega [B,T,H,N] fp32 (per token); u [H,N] fp32; s_in, gs_out [B,H,N,N] fp32 or
    None.  Returns (gr, gk, gv, gomega [B,T,H,N], gu [H,N]) and, with ``want_gs_in``, the gradient
    of s_in as well."""
    import torch

    _need_cuda(r, k, v, omega, u, gy, s_in, gs_out)
    B, T, H, N = r.shape
    for t in (r, k, v, gy):
        if t.dtype != torch.bfloat16 or t.shape != r.shape:
            raise ValueError("r, k, v, gy must be bf16 of the same shape")
    _f32("omega", omega, B * T * H * N)
    _f32("u", u, H * N)
    for name, t in (("s_in", s_in), ("gs_out", gs_out)):
        if t is not None:
            _f32(name, t, B * H * N * N)
    h = lib()
    gr, gk, gv = torch.empty_like(r), torch.empty_like(k), torch.empty_like(v)
    gomega = torch.empty((B, T, H, N), dtype=torch.float32, device=r.device)
    gu = torch.empty((H, N), dtype=torch.float32, device=r.device)
    gsi = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device) if want_gs_in else None
    wsb = int(h.rwkv_wkv6_backward_workspace_bytes(B, T, H, N))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=r.device)
    _check("rwkv_wkv6_backward",
           h.rwkv_wkv6_backward(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(s_in), _ptr(gy),
                                _ptr(gs_out), _ptr(gr), _ptr(gk), _ptr(gv), _ptr(gomega), _ptr(gu), _ptr(gsi),
                                _ptr(ws), wsb, _stream(stream)))
    res = (gr, gk, gv, gomega, gu)
    return res + (gsi,) if want_gs_in else res


def rwkv_wkv5_step(r, k, v, omega, u, state=None, *, state_out=None, stream=None, out=None):
    """Eagle / RWKV-5 decode step: r, k, v [B,H,N] bf16 (one token per stream);
    omega, u [H,N] fp32; state [B,H,N,N] fp32 or None (zero).  Returns
    (y [B,H,N] bf16, new state).  state_out may be `state` (in-place)."""
    import torch

    _need_cuda(r, k, v, omega, u, state, state_out)
    B, H, N = r.shape
    for t in (r, k, v):
        if t.dtype != torch.bfloat16 or t.shape != r.shape:
            raise ValueError("r, k, v must be bf16 of the same shape")
    _f32("omega", omega, H * N)
    _f32("u", u, H * N)
    y = torch.empty_like(r) if out is None else out
    so = state_out if state_out is not None else torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    _check("rwkv_wkv5_step",
           lib().rwkv_wkv5_step(B, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(y), _ptr(state),
                                _ptr(so), _stream(stream)))
    return y, so


# ------------------------------------------------------------------ WKV-6
def rwkv_wkv6_forward(r, k, v, omega, u, s_in=None, *, return_state=False, stream=None, out=None):
    """Finch / RWKV-6 forward (per-token decay): r, k, v [B,T,H,N] bf16;
    omega [B,T,H,N] fp32; u [H,N] fp32; s_in [B,H,N,N] fp32 or None."""
    import torch

    _need_cuda(r, k, v, omega, u, s_in)
    B, T, H, N = r.shape
    for t in (r, k, v):
        if t.dtype != torch.bfloat16 or t.shape != r.shape:
            raise ValueError("r, k, v must be bf16 of the same shape")
    if omega.dtype != torch.float32 or omega.shape != r.shape or not omega.is_contiguous():
        raise ValueError("omega must be a contiguous float32 tensor shaped like r")
    _f32("u", u, H * N)
    h = lib()
    y = torch.empty_like(r) if out is None else out
    so = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device) if return_state else None
    wsb = int(h.rwkv_wkv6_forward_workspace_bytes(B, T, H, N))
    ws = torch.empty(wsb, dtype=torch.uint8, device=r.device) if wsb else None
    _check("rwkv_wkv6_forward",
           h.rwkv_wkv6_forward(B, T, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(y),
                               _ptr(s_in), _ptr(so), _ptr(ws), wsb, _stream(stream)))
    return (y, so) if return_state else y


def rwkv_wkv6_step(r, k, v, omega, u, state=None, *, state_out=None, stream=None, out=None):
    """Finch / RWKV-6 decode step: r, k, v [B,H,N] bf16 and omega [B,H,N] fp32
    (one token per stream); u [H,N] fp32; state [B,H,N,N] fp32 or None (zero).
    Returns (y [B,H,N] bf16, new state).  state_out may be `state` (in-place)."""
    import torch

    _need_cuda(r, k, v, omega, u, state, state_out)
    B, H, N = r.shape
    for t in (r, k, v):
        if t.dtype != torch.bfloat16 or t.shape != r.shape:
            raise ValueError("r, k, v must be bf16 of the same shape")
    _f32("omega", omega, B * H * N)
    _f32("u", u, H * N)
    y = torch.empty_like(r) if out is None else out
    so = state_out if state_out is not None else torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    _check("rwkv_wkv6_step",
           lib().rwkv_wkv6_step(B, H, N, _ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(y), _ptr(state),
                                _ptr(so), _stream(stream)))
    return y, so


def rwkv_check_device_error(stream=None):
    """Synchronise the stream and raise if a kernel's bounded wait timed out."""
    _check("rwkv_check_device_error", lib().rwkv_check_device_error(_stream(stream)))

