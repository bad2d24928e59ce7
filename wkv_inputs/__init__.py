"""Seeded synthetic inputs for the WKV operator: the one module that both the
fp64 oracle (through the tests) and the CUDA path read their inputs from.

It holds none of the operator's arithmetic.  It only draws numbers with the
distributions that the WKV workloads use:

* RWKV-4 WKV: per-channel decay rate ``w`` log-uniform on [0.01, 5], bonus
  ``u ~ U(-1, 1)``, keys and values ``k, v ~ N(0, 1)`` i.i.d., optionally 1 % of
  the keys replaced by ``±U(20, 40)`` outliers, upstream gradient
  ``gy ~ N(0, 1)``; with the receptance gate, ``r ~ N(0, 1)`` and the upstream
  gradient of the gated output ``go ~ N(0, 1)``.
* Eagle / RWKV-5 WKV: ``r, k, v ~ N(0, 1)/sqrt(N)`` rounded to bf16, per-channel
  ``omega ~ U(-6, 0)`` and ``u ~ U(-1, 1)`` of shape ``[H, N]``.
* Finch / RWKV-6 WKV: as Eagle, with a per-token decay parameter
  ``omega[b, t, h, n] = omega0[h, n] + 0.5 * z`` (fp32), a per-channel base
  ``omega0 ~ U(-6, 0)`` plus an i.i.d. ``z ~ N(0, 1)`` per token: the
  input-dependent correction of the decay around a learned per-channel value.

Generator.  Every value is a pure function of ``(seed, tensor id, flat
index)``: the SplitMix64 finaliser (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) hashes a per-tensor key plus
``(index + 1)`` times the golden-ratio increment, the top 53 bits give a double
in [0, 1), and normals come from the Box-Muller transform.  So any sub-block of
a tensor (a time slice, a sample of lanes) regenerates on its own with the same
values, on the CPU or on a CUDA device.  Integer hashing is bit-identical on
both devices; the Box-Muller ``log``/``cos`` may differ in the last bit between
devices, so a test that compares two implementations generates once and hands
both sides the same bytes.
"""

from __future__ import annotations

import math

import torch

__all__ = [
    "splitmix64_scalar",
    "uniform",
    "normal",
    "TID",
    "btc_field",
    "wkv4_params",
    "wkv4_problem",
    "wkv5_problem",
    "wkv6_problem",
    "CONFIG_SEED_BASE",
]

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB

# Default seed of workload i is CONFIG_SEED_BASE + i.
CONFIG_SEED_BASE = 20261202

# Tensor ids: each named input draws from its own stream.
TID = {
    "w": 1,
    "u": 2,
    "k": 3,
    "v": 4,
    "gy": 5,
    "r": 6,
    "omega": 7,
    "k_outlier": 8,
    "omega_t": 9,
    "s_in": 10,
    "gs_out": 11,
}


def _s64(x: int) -> int:
    """Unsigned 64-bit pattern -> the signed int64 with the same bits."""
    x &= _M64
    return x - (1 << 64) if x >= (1 << 63) else x


def splitmix64_scalar(z: int) -> int:
    """SplitMix64 finaliser on a Python int (unsigned 64-bit semantics)."""
    z &= _M64
    z = ((z ^ (z >> 30)) * _C1) & _M64
    z = ((z ^ (z >> 27)) * _C2) & _M64
    return z ^ (z >> 31)


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    # int64 products wrap modulo 2^64, which is the unsigned product's low half.
    z = (z ^ _lsr(z, 30)) * _s64(_C1)
    z = (z ^ _lsr(z, 27)) * _s64(_C2)
    return z ^ _lsr(z, 31)


def _key(seed: int, tid: int, sub: int) -> int:
    """Per-(seed, tensor, sub-stream) 64-bit key."""
    h = splitmix64_scalar(seed * _GAMMA + 0x632BE59BD9B4E019)
    h = splitmix64_scalar(h ^ (tid * 0xD1B54A32D192ED03))
    h = splitmix64_scalar(h ^ (sub * 0x8CB92BA72F3D8DD7 + 1))
    return h


def _bits(seed: int, tid: int, sub: int, idx: torch.Tensor) -> torch.Tensor:
    key = _s64(_key(seed, tid, sub))
    z = key + (idx + 1) * _s64(_GAMMA)
    return _mix(z)


def uniform(seed: int, tid: int, idx: torch.Tensor, sub: int = 0) -> torch.Tensor:
    """U[0, 1) doubles, one per entry of the int64 index tensor ``idx``."""
    b = _bits(seed, tid, sub, idx)
    return _lsr(b, 11).to(torch.float64) * (2.0 ** -53)


def normal(seed: int, tid: int, idx: torch.Tensor) -> torch.Tensor:
    """N(0, 1) doubles by Box-Muller on two independent uniform sub-streams."""
    u1 = uniform(seed, tid, idx, sub=0)
    u2 = uniform(seed, tid, idx, sub=1)
    rad = torch.sqrt(-2.0 * torch.log1p(-u1))  # 1 - u1 in (0, 1]
    return rad * torch.cos((2.0 * math.pi) * u2)


def _index_btc(B: int, T: int, C: int, t0: int, t1: int, b_sel, c_sel, device, b0=0, b1=None):
    """Flat indices (b*T + t)*C + c of the [B, T, C] tensor for t in [t0, t1).

    Without a selection the result is [b1-b0, t1-t0, C] for batch rows
    [b0, b1); with ``b_sel``/``c_sel`` (equal-length 1-D index tensors naming
    lanes) it is [t1-t0, n_lanes].
    """
    t = torch.arange(t0, t1, device=device, dtype=torch.int64)
    if b_sel is None:
        b1 = B if b1 is None else b1
        b = torch.arange(b0, b1, device=device, dtype=torch.int64).view(-1, 1, 1)
        c = torch.arange(C, device=device, dtype=torch.int64).view(1, 1, C)
        return (b * T + t.view(1, -1, 1)) * C + c
    b_sel = torch.as_tensor(b_sel, dtype=torch.int64, device=device).view(1, -1)
    c_sel = torch.as_tensor(c_sel, dtype=torch.int64, device=device).view(1, -1)
    return (b_sel * T + t.view(-1, 1)) * C + c_sel


def btc_field(kind: str, seed: int, B: int, T: int, C: int, t0: int = 0, t1=None,
              b_sel=None, c_sel=None, outliers: bool = False,
              dtype=torch.float32, device="cpu", block: int = 1 << 23,
              b0: int = 0, b1=None) -> torch.Tensor:
    """A [B, T, C] input (k, v or gy) restricted to time steps [t0, t1) and
    batch rows [b0, b1) (or to the lanes ``b_sel``, ``c_sel``).

    ``outliers`` replaces each key, independently with probability 0.01, by
    ``s * U(20, 40)`` with a fair random sign ``s`` (the heavy-tailed keys that
    exercise the running-max stabilisation of the WKV scan).
    """
    t1 = T if t1 is None else t1
    tid = TID[kind]
    idx = _index_btc(B, T, C, t0, t1, b_sel, c_sel, device, b0, b1)
    flat = idx.reshape(-1)
    out = torch.empty(flat.numel(), dtype=dtype, device=device)
    for s in range(0, flat.numel(), block):
        ix = flat[s:s + block]
        val = normal(seed, tid, ix)
        if outliers:
            pick = uniform(seed, TID["k_outlier"], ix, sub=0) < 0.01
            sign = torch.where(uniform(seed, TID["k_outlier"], ix, sub=1) < 0.5, -1.0, 1.0)
            mag = 20.0 + 20.0 * uniform(seed, TID["k_outlier"], ix, sub=2)
            val = torch.where(pick, sign * mag, val)
        out[s:s + block] = val.to(dtype)
    return out.view(idx.shape)


def wkv4_params(seed: int, C: int, c_sel=None, device="cpu"):
    """Per-channel (w, u), float32: w log-uniform on [0.01, 5], u ~ U(-1, 1)."""
    c = torch.arange(C, dtype=torch.int64, device=device) if c_sel is None else \
        torch.as_tensor(c_sel, dtype=torch.int64, device=device)
    lo, hi = math.log(0.01), math.log(5.0)
    w = torch.exp(lo + (hi - lo) * uniform(seed, TID["w"], c))
    u = -1.0 + 2.0 * uniform(seed, TID["u"], c)
    return w.to(torch.float32), u.to(torch.float32)


def wkv4_problem(B: int, T: int, C: int, seed: int, outliers: bool = False,
                 with_gy: bool = False, dtype=torch.float32, device="cpu", gated: bool = False) -> dict:
    """Full RWKV-4 WKV inputs: w, u [C] fp32; k, v (and gy) [B, T, C] of ``dtype``;
    with ``gated``, also the receptance r and (with ``with_gy``) the gradient
    ``go`` of the gated output [B, T, C] (``go`` is drawn from gy's stream)."""
    w, u = wkv4_params(seed, C, device=device)
    p = {
        "w": w,
        "u": u,
        "k": btc_field("k", seed, B, T, C, outliers=outliers, dtype=dtype, device=device),
        "v": btc_field("v", seed, B, T, C, dtype=dtype, device=device),
    }
    if with_gy:
        p["go" if gated else "gy"] = btc_field("gy", seed, B, T, C, dtype=dtype, device=device)
    if gated:
        p["r"] = btc_field("r", seed, B, T, C, dtype=dtype, device=device)
    return p


def wkv5_problem(B: int, T: int, H: int, N: int, seed: int, device="cpu",
                 omega_range=(-6.0, 0.0)) -> dict:
    """Eagle / RWKV-5 WKV inputs.

    r, k, v: [B, T, H, N] bf16, N(0, 1)/sqrt(N) rounded to nearest even;
    omega: [H, N] fp32 ~ U(omega_range); u: [H, N] fp32 ~ U(-1, 1).
    """
    n = B * T * H * N
    idx = torch.arange(n, dtype=torch.int64, device=device)
    scale = 1.0 / math.sqrt(N)
    out = {}
    for name in ("r", "k", "v"):
        val = torch.empty(n, dtype=torch.bfloat16, device=device)
        blk = 1 << 23
        for s in range(0, n, blk):
            val[s:s + blk] = (normal(seed, TID[name], idx[s:s + blk]) * scale).to(torch.bfloat16)
        out[name] = val.view(B, T, H, N)
    hn = torch.arange(H * N, dtype=torch.int64, device=device)
    lo, hi = omega_range
    out["omega"] = (lo + (hi - lo) * uniform(seed, TID["omega"], hn)).to(torch.float32).view(H, N)
    out["u"] = (-1.0 + 2.0 * uniform(seed, TID["u"], hn)).to(torch.float32).view(H, N)
    return out


def wkv6_problem(B: int, T: int, H: int, N: int, seed: int, device="cpu",
                 omega_range=(-6.0, 0.0), omega_jitter: float = 0.5) -> dict:
    """Finch / RWKV-6 WKV inputs: the Eagle inputs of ``wkv5_problem`` with the
    per-channel ``omega`` [H, N] widened to a per-token ``omega`` [B, T, H, N]
    fp32: ``omega0[h, n] + omega_jitter * N(0, 1)``."""
    out = wkv5_problem(B, T, H, N, seed, device=device, omega_range=omega_range)
    base = out["omega"]
    n = B * T * H * N
    om = torch.empty(n, dtype=torch.float32, device=device)
    blk = 1 << 23
    for s in range(0, n, blk):
        ix = torch.arange(s, min(n, s + blk), dtype=torch.int64, device=device)
        om[s:s + blk] = (base.reshape(-1)[ix % (H * N)].double() +
                         omega_jitter * normal(seed, TID["omega_t"], ix)).to(torch.float32)
    out["omega"] = om.view(B, T, H, N)
    return out


def wkv5_grads(B: int, T: int, H: int, N: int, seed: int, device="cpu", states: bool = False) -> dict:
    """Upstream gradients for the Eagle / Finch backward: gy [B, T, H, N] bf16 ~ N(0, 1) (rounded
    to nearest even); with ``states``, an initial state s_in and a final-state gradient gs_out,
    [B, H, N, N] fp32 ~ N(0, 1)/N (the scale of a state built from N(0,1)/sqrt(N) keys and values)."""
    n = B * T * H * N
    idx = torch.arange(n, dtype=torch.int64, device=device)
    gy = torch.empty(n, dtype=torch.bfloat16, device=device)
    blk = 1 << 23
    for s in range(0, n, blk):
        gy[s:s + blk] = normal(seed, TID["gy"], idx[s:s + blk]).to(torch.bfloat16)
    out = {"gy": gy.view(B, T, H, N)}
    if states:
        m = torch.arange(B * H * N * N, dtype=torch.int64, device=device)
        for name in ("s_in", "gs_out"):
            out[name] = (normal(seed, TID[name], m) / N).to(torch.float32).view(B, H, N, N)
    return out
