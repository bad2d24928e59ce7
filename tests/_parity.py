"""Comparison rules shared by the GPU parity tests.

Tolerances (stated once, used everywhere):
* fp32 WKV-4 outputs:      |got - ref| <= 1e-5 * max(1, |ref|)
* fp32 WKV-4 gradients gk, gv, gw, gu (and gr of the gated operator):
                           |got - ref| <= 1e-4 * max(1, |ref|) elementwise;
  for gw, gu (each entry a sum over B*T terms) the norm-wise ratio
  max |got - ref| / max(1, max |ref|) is reported beside it.  Where a test
  passes the entries' conditioning floor (wkv4_input_sensitivity), an entry's
  bound is at least twice the movement of the oracle's own result under
  half-ulp perturbations of the fp32 inputs
* bf16 I/O (fp32 inside):  |got - ref| <= 8e-3 * max(|ref|, rms(ref))
  (rms over the compared tensor; a bf16 output alone is rounded by <= 2^-9 relative)
* WKV-4 states compare through a/b (1e-5 * max(1, |A/B|)) and log2 b + p
  (2e-5 absolute), because (a, b, p) is defined only up to a power of two.
"""
import numpy as np
import torch

TOL_Y = 1e-5
TOL_GRAD = 1e-4
TOL_BF16 = 8e-3


def _np(x):
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu()
        if x.dtype == torch.bfloat16:
            x = x.float()
        return x.double().numpy()
    return np.asarray(x, dtype=np.float64)


def assert_close_abs1(got, ref, tol, what=""):
    """|got - ref| <= tol * max(1, |ref|) elementwise."""
    g, r = _np(got), _np(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    bound = tol * np.maximum(1.0, np.abs(r))
    err = np.abs(g - r)
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), (f"{what}: max |err|/bound = {np.max(err / bound):.3g} at {worst}: "
                                  f"got {g[worst]!r} ref {r[worst]!r}")
    return float(np.max(err / bound))


def assert_close_normwise(got, ref, tol, what=""):
    """max |got - ref| <= tol * max(1, max |ref|): relative error of a vector of
    reductions, measured against its largest entry."""
    g, r = _np(got), _np(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    bound = tol * max(1.0, float(np.max(np.abs(r))))
    err = float(np.max(np.abs(g - r)))
    assert err <= bound, f"{what}: max |err| = {err:.3g} > {bound:.3g} (norm-wise)"
    return err / bound


def normwise_ratio(got, ref):
    """max |got - ref| / max(1, max |ref|): the error of a vector of reductions against its
    largest entry (reported beside the elementwise check, not a looser bound)."""
    g, r = _np(got), _np(ref)
    return float(np.max(np.abs(g - r))) / max(1.0, float(np.max(np.abs(r))))


def assert_grads_close(got, ref, what="", names=("gk", "gv", "gw", "gu"), floor=None):
    """Gradients against the oracle, every one elementwise: |got - ref| <= 1e-4 max(1, |ref|).
    ``floor`` maps a name to per-element conditioning floors (wkv4_input_sensitivity): where the
    oracle's own result moves by more than the bound under half-ulp perturbations of the fp32
    inputs, no fp32 computation can do better, and the bound becomes twice that movement.
    Returns the worst elementwise error/bound ratio and, for gw and gu, the norm-wise ratio and
    the number of entries on the floor."""
    report = {}
    for g, r, name in zip(got, ref, names):
        fl = None if floor is None else floor.get(name)
        if fl is None:
            report[name] = assert_close_abs1(g, r, TOL_GRAD, f"{what}{name}")
        else:
            gg, rr = _np(g), _np(r)
            assert np.all(np.isfinite(gg)), f"{what}{name}: non-finite GPU values"
            base = TOL_GRAD * np.maximum(1.0, np.abs(rr))
            bound = np.maximum(base, 2.0 * np.asarray(fl, dtype=np.float64))
            err = np.abs(gg - rr)
            worst = int(np.argmax(err / bound))
            assert np.all(err <= bound), (f"{what}{name}: max |err|/bound = {np.max(err / bound):.3g} at {worst}: "
                                          f"got {gg.flat[worst]!r} ref {rr.flat[worst]!r} floor {fl.flat[worst]!r}")
            report[name] = float(np.max(err / bound))
            report[name + "_on_floor"] = int(np.sum(bound > base))
            report[name + "_vs_1e-4"] = float(np.max(err / base))
        if name in ("gw", "gu"):
            report[name + "_normwise"] = normwise_ratio(g, r)
    print(f"{what}gradient error / bound: " + ", ".join(f"{k} {v:.3g}" for k, v in report.items()))
    return report


def wkv4_input_sensitivity(oracle, w, u, k, v, gy, trials=2, seed=0):
    """How far the fp64 oracle's gw and gu move when every fp32 input (w, u, k, v, gy) is
    perturbed by up to half an ulp (relative 2^-24), max over a few random perturbations:
    the conditioning floor of each entry, the error any fp32 computation of it may carry."""
    rng = np.random.default_rng(seed)
    ins = [_np(x) for x in (w, u, k, v, gy)]
    _, _, gw0, gu0 = oracle.wkv4_backward(*ins)
    dw, du = np.zeros_like(gw0), np.zeros_like(gu0)
    for _ in range(trials):
        pert = [x * (1.0 + rng.uniform(-2.0 ** -24, 2.0 ** -24, x.shape)) for x in ins]
        _, _, gw1, gu1 = oracle.wkv4_backward(*pert)
        dw = np.maximum(dw, np.abs(gw1 - gw0))
        du = np.maximum(du, np.abs(gu1 - gu0))
    return {"gw": dw, "gu": du}


def assert_close_rms(got, ref, tol, what=""):
    """|got - ref| <= tol * max(|ref|, rms(ref)) elementwise."""
    g, r = _np(got), _np(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    rms = float(np.sqrt(np.mean(r * r)))
    bound = tol * np.maximum(np.abs(r), rms)
    err = np.abs(g - r)
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), (f"{what}: max |err|/bound = {np.max(err / bound):.3g} at {worst}: "
                                  f"got {g[worst]!r} ref {r[worst]!r}")
    return float(np.max(err / bound))


def assert_state_close(gpu_state, ref_ab, what="state"):
    """gpu_state [3,...] = (a, b, p); ref_ab [2,...] = (A, B) in fp64."""
    s = _np(gpu_state)
    r = _np(ref_ab)
    a, b, p = s[0], s[1], s[2]
    assert_close_abs1(a / b, r[0] / r[1], TOL_Y, what + " a/b")
    lg = np.log2(b) + p
    lr = np.log2(r[1])
    assert np.all(np.abs(lg - lr) <= 2e-5), f"{what}: log2 b + p off by {np.max(np.abs(lg - lr)):.3g}"


def sample_lanes(B, C, n, seed=0):
    """n distinct (b, c) lanes, reproducibly."""
    rng = np.random.default_rng(seed)
    flat = rng.choice(B * C, size=min(n, B * C), replace=False)
    return torch.from_numpy(flat // C), torch.from_numpy(flat % C)


def state_to_ab(state):
    """(a, b, p) planes -> float64 (A, B) = (a 2^p, b 2^p), for comparisons."""
    s = state.double()
    scale = torch.pow(2.0, s[2])
    return torch.stack([s[0] * scale, s[1] * scale])
