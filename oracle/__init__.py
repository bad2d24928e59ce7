"""fp64 CPU oracle for the RWKV WKV operator (Python face of ``wkv_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg call this; the CUDA library and its Python binding
never import it.  Every function takes array-likes (numpy arrays or CPU torch
tensors of any float dtype, widened exactly to float64) and returns float64
numpy arrays.  The C source cites the formula each function follows.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, invariants, brute force and finite differences.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``wkv_oracle.c`` into ``liboracle.so`` (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        sigs = {
            "oracle_wkv4_forward": [I, I, I, P, P, P, P, P, P, P],
            "oracle_wkv4_forward_bruteforce": [I, I, I, P, P, P, P, P],
            "oracle_wkv4_backward": [I, I, I, P, P, P, P, P, P, P, P, P, P],
            "oracle_wkv4_backward_bruteforce": [I, I, I, P, P, P, P, P, P, P, P, P],
            "oracle_wkv4_step": [I, I, P, P, P, P, P, P],
            "oracle_wkv5_forward": [I, I, I, I, P, P, P, P, P, P, P, P],
            "oracle_wkv5_forward_bruteforce": [I, I, I, I, P, P, P, P, P, P],
            "oracle_wkv6_forward": [I, I, I, I, P, P, P, P, P, P, P, P],
            "oracle_wkv4_gated_forward": [I, I, I, P, P, P, P, P, P, P, P],
            "oracle_wkv5_backward": [I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
            "oracle_wkv6_backward": [I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
            "oracle_wkv4_gated_backward": [I, I, I, P, P, P, P, P, P, P, P, P, P, P, P],
            "oracle_wkv6_forward_bruteforce": [I, I, I, I, P, P, P, P, P, P],
        }
        for name, args in sigs.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int64
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """Runs later oracle calls on n OpenMP threads; returns the count in force."""
    return int(_load().oracle_set_num_threads(int(n)))


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleNonFinite(RuntimeError):
    """The oracle produced a non-finite output (an overflow of the fp64 form)."""


def _check(nbad, name):
    if nbad:
        raise OracleNonFinite(f"{name}: {nbad} non-finite outputs")


def wkv4_forward(w, u, k, v, state_in=None, return_state=False):
    """WKV-4 forward by the recurrent form.  k, v [B,T,C]; w, u [C];
    state_in [2,B,C] = (a, b) or None.  Returns y [B,T,C] (and state [2,B,C])."""
    lib = _load()
    w, u, k, v, s0 = map(_f64, (w, u, k, v, state_in))
    B, T, C = k.shape
    y = np.empty((B, T, C))
    s1 = np.empty((2, B, C))
    _check(lib.oracle_wkv4_forward(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(s0), _p(y), _p(s1)),
           "wkv4_forward")
    return (y, s1) if return_state else y


def wkv4_forward_bruteforce(w, u, k, v):
    """WKV-4 forward by the O(T^2) time-parallel form, zero initial state."""
    lib = _load()
    w, u, k, v = map(_f64, (w, u, k, v))
    B, T, C = k.shape
    y = np.empty((B, T, C))
    _check(lib.oracle_wkv4_forward_bruteforce(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(y)),
           "wkv4_forward_bruteforce")
    return y


def wkv4_backward(w, u, k, v, gy, state_in=None):
    """WKV-4 gradients of sum(gy * y): returns (gk, gv, gw, gu); gw, gu [C]
    summed over batch and time."""
    lib = _load()
    w, u, k, v, gy, s0 = map(_f64, (w, u, k, v, gy, state_in))
    B, T, C = k.shape
    gk = np.empty((B, T, C))
    gv = np.empty((B, T, C))
    gw = np.empty(C)
    gu = np.empty(C)
    _check(lib.oracle_wkv4_backward(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(gy), _p(s0),
                                    _p(gk), _p(gv), _p(gw), _p(gu)), "wkv4_backward")
    return gk, gv, gw, gu


def wkv4_backward_bruteforce(w, u, k, v, gy):
    """WKV-4 gradients from the O(T^2) time-parallel form, zero initial state."""
    lib = _load()
    w, u, k, v, gy = map(_f64, (w, u, k, v, gy))
    B, T, C = k.shape
    gk = np.empty((B, T, C))
    gv = np.empty((B, T, C))
    gw = np.empty(C)
    gu = np.empty(C)
    _check(lib.oracle_wkv4_backward_bruteforce(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(gy),
                                               _p(gk), _p(gv), _p(gw), _p(gu)),
           "wkv4_backward_bruteforce")
    return gk, gv, gw, gu


def wkv4_step(w, u, k, v, state):
    """One recurrent step: k, v [B,C]; state [2,B,C] (a, b).  Returns (y, new_state)."""
    lib = _load()
    w, u, k, v = map(_f64, (w, u, k, v))
    st = _f64(state).copy()
    B, C = k.shape
    y = np.empty((B, C))
    _check(lib.oracle_wkv4_step(B, C, _p(w), _p(u), _p(k), _p(v), _p(st), _p(y)), "wkv4_step")
    return y, st


def wkv5_forward(r, k, v, omega, u, s_in=None, return_state=False):
    """Eagle / RWKV-5 WKV forward.  r, k, v [B,T,H,N]; omega, u [H,N];
    s_in [B,H,N,N] or None.  Returns y [B,T,H,N] (and s_out [B,H,N,N])."""
    lib = _load()
    r, k, v, omega, u, s0 = map(_f64, (r, k, v, omega, u, s_in))
    B, T, H, N = r.shape
    y = np.empty((B, T, H, N))
    s1 = np.empty((B, H, N, N))
    _check(lib.oracle_wkv5_forward(B, T, H, N, _p(r), _p(k), _p(v), _p(omega), _p(u), _p(s0),
                                   _p(y), _p(s1)), "wkv5_forward")
    return (y, s1) if return_state else y


def wkv5_forward_bruteforce(r, k, v, omega, u):
    """Eagle / RWKV-5 WKV forward as an explicit sum over past tokens, zero state."""
    lib = _load()
    r, k, v, omega, u = map(_f64, (r, k, v, omega, u))
    B, T, H, N = r.shape
    y = np.empty((B, T, H, N))
    _check(lib.oracle_wkv5_forward_bruteforce(B, T, H, N, _p(r), _p(k), _p(v), _p(omega), _p(u),
                                              _p(y)), "wkv5_forward_bruteforce")
    return y


def wkv6_forward(r, k, v, omega, u, s_in=None, return_state=False):
    """Finch / RWKV-6 WKV forward (per-token decay).  r, k, v, omega [B,T,H,N];
    u [H,N]; s_in [B,H,N,N] or None.  Returns y [B,T,H,N] (and s_out [B,H,N,N])."""
    lib = _load()
    r, k, v, omega, u, s0 = map(_f64, (r, k, v, omega, u, s_in))
    B, T, H, N = r.shape
    y = np.empty((B, T, H, N))
    s1 = np.empty((B, H, N, N))
    _check(lib.oracle_wkv6_forward(B, T, H, N, _p(r), _p(k), _p(v), _p(omega), _p(u), _p(s0),
                                   _p(y), _p(s1)), "wkv6_forward")
    return (y, s1) if return_state else y


def wkv6_forward_bruteforce(r, k, v, omega, u):
    """Finch / RWKV-6 WKV forward as an explicit sum over past tokens with the
    decay products formed term by term, zero state."""
    lib = _load()
    r, k, v, omega, u = map(_f64, (r, k, v, omega, u))
    B, T, H, N = r.shape
    y = np.empty((B, T, H, N))
    _check(lib.oracle_wkv6_forward_bruteforce(B, T, H, N, _p(r), _p(k), _p(v), _p(omega), _p(u),
                                              _p(y)), "wkv6_forward_bruteforce")
    return y


def wkv4_gated_forward(w, u, k, v, r, state_in=None, return_state=False):
    """Receptance-gated WKV-4 forward o = sigmoid(r) * WKV.  k, v, r [B,T,C];
    w, u [C]; state_in [2,B,C] or None.  Returns o (and the state [2,B,C])."""
    lib = _load()
    w, u, k, v, r, s0 = map(_f64, (w, u, k, v, r, state_in))
    B, T, C = k.shape
    o = np.empty((B, T, C))
    s1 = np.empty((2, B, C))
    _check(lib.oracle_wkv4_gated_forward(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(r), _p(s0), _p(o), _p(s1)),
           "wkv4_gated_forward")
    return (o, s1) if return_state else o


def wkv4_gated_backward(w, u, k, v, r, go, state_in=None):
    """Gradients of sum(go * o) for the gated forward: (gk, gv, gr, gw, gu)."""
    lib = _load()
    w, u, k, v, r, go, s0 = map(_f64, (w, u, k, v, r, go, state_in))
    B, T, C = k.shape
    gk, gv, gr = np.empty((B, T, C)), np.empty((B, T, C)), np.empty((B, T, C))
    gw, gu = np.empty(C), np.empty(C)
    _check(lib.oracle_wkv4_gated_backward(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(r), _p(go), _p(s0),
                                          _p(gk), _p(gv), _p(gr), _p(gw), _p(gu)), "wkv4_gated_backward")
    return gk, gv, gr, gw, gu


def _wkv56_backward(fn, name, r, k, v, omega, u, gy, s_in=None, gs_out=None, per_token=False):
    lib = _load()
    r, k, v, omega, u, gy, s0, gso = map(_f64, (r, k, v, omega, u, gy, s_in, gs_out))
    B, T, H, N = r.shape
    gr, gk, gv = np.empty((B, T, H, N)), np.empty((B, T, H, N)), np.empty((B, T, H, N))
    gom = np.empty((B, T, H, N) if per_token else (H, N))
    gu = np.empty((H, N))
    gsi = np.empty((B, H, N, N))
    _check(getattr(lib, fn)(B, T, H, N, _p(r), _p(k), _p(v), _p(omega), _p(u), _p(s0), _p(gy), _p(gso),
                            _p(gr), _p(gk), _p(gv), _p(gom), _p(gu), _p(gsi)), name)
    return gr, gk, gv, gom, gu, gsi


def wkv5_backward(r, k, v, omega, u, gy, s_in=None, gs_out=None):
    """Gradients of sum(gy * y) + sum(gs_out * s_out) for the Eagle forward: returns
    (gr, gk, gv, gomega [H,N], gu [H,N], gs_in [B,H,N,N])."""
    return _wkv56_backward("oracle_wkv5_backward", "wkv5_backward", r, k, v, omega, u, gy, s_in, gs_out)


def wkv6_backward(r, k, v, omega, u, gy, s_in=None, gs_out=None):
    """Gradients of sum(gy * y) + sum(gs_out * s_out) for the Finch forward: returns
    (gr, gk, gv, gomega [B,T,H,N], gu [H,N], gs_in [B,H,N,N])."""
    return _wkv56_backward("oracle_wkv6_backward", "wkv6_backward", r, k, v, omega, u, gy, s_in, gs_out,
                           per_token=True)
