"""Pins for the fp64 backward of the Eagle / RWKV-5 and Finch / RWKV-6 forwards
(the pages print no backward; the oracle takes the chain rule through the
recurrence).  Each pin checks it against something other than its own code:
central finite differences of L = sum(gy * y) + sum(gs_out * s_out) for every
input, and the time-reversal identity that makes gv and the gradient of the
initial state a forward of the operator itself (pinned on its own) run
backwards in time with the roles of r and k swapped and gy as the value."""
import numpy as np
import pytest

import oracle
import wkv_inputs as wi


def _problem(finch, B, T, H, N, seed, omega_range=(-2.0, 0.5)):
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    p = {k: v.double().numpy() for k, v in gen(B, T, H, N, seed, omega_range=omega_range).items()}
    rng = np.random.default_rng(seed)
    p["gy"] = rng.standard_normal(p["r"].shape)
    p["s_in"] = rng.standard_normal((B, H, N, N))
    p["gs_out"] = rng.standard_normal((B, H, N, N))
    return p


def _fwd(finch):
    return oracle.wkv6_forward if finch else oracle.wkv5_forward


def _bwd(finch):
    return oracle.wkv6_backward if finch else oracle.wkv5_backward


@pytest.mark.parametrize("finch", [False, True])
def test_backward_matches_finite_differences(finch):
    B, T, H, N, h = 1, 6, 2, 3, 1e-6
    p = _problem(finch, B, T, H, N, 71)

    def loss(q):
        y, s = _fwd(finch)(q["r"], q["k"], q["v"], q["omega"], q["u"], s_in=q["s_in"], return_state=True)
        return float(np.sum(p["gy"] * y) + np.sum(p["gs_out"] * s))

    gr, gk, gv, gom, gu, gsi = _bwd(finch)(p["r"], p["k"], p["v"], p["omega"], p["u"], p["gy"], s_in=p["s_in"],
                                           gs_out=p["gs_out"])
    for name, grad in (("r", gr), ("k", gk), ("v", gv), ("omega", gom), ("u", gu), ("s_in", gsi)):
        num = np.zeros_like(p[name])
        for idx in np.ndindex(p[name].shape):
            qp = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
            qm = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
            qp[name][idx] += h
            qm[name][idx] -= h
            num[idx] = (loss(qp) - loss(qm)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("finch", [False, True])
def test_value_gradient_is_the_forward_run_backwards(finch):
    # Without gs_out, gv_s[j] = sum_{t>s} (sum_i r_t[i] * decay(s -> t)_i * k_s[i]) gy_t[j] + bonus_s gy_s[j]:
    # the forward over the reversed sequence with r <- k, k <- r, v <- gy (the decays between two tokens
    # are the same set either way).  Its final state is the gradient of the initial state.
    B, T, H, N = 2, 24, 2, 8
    p = _problem(finch, B, T, H, N, 72)
    rev = lambda x: np.ascontiguousarray(x[:, ::-1])
    om_rev = rev(p["omega"]) if finch else p["omega"]
    y_rev, s_rev = _fwd(finch)(rev(p["k"]), rev(p["r"]), rev(p["gy"]), om_rev, p["u"], return_state=True)
    _, _, gv, _, _, gsi = _bwd(finch)(p["r"], p["k"], p["v"], p["omega"], p["u"], p["gy"], s_in=p["s_in"])
    np.testing.assert_allclose(gv, rev(y_rev), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gsi, s_rev, rtol=1e-12, atol=1e-13)


def test_finch_backward_with_constant_decay_is_eagle():
    B, T, H, N = 1, 20, 2, 6
    p = _problem(False, B, T, H, N, 73)
    om_t = np.broadcast_to(p["omega"][None, None], (B, T, H, N)).copy()
    e = oracle.wkv5_backward(p["r"], p["k"], p["v"], p["omega"], p["u"], p["gy"], s_in=p["s_in"],
                             gs_out=p["gs_out"])
    f = oracle.wkv6_backward(p["r"], p["k"], p["v"], om_t, p["u"], p["gy"], s_in=p["s_in"], gs_out=p["gs_out"])
    for a, b in zip(e[:3] + e[4:], f[:3] + f[4:]):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    # the per-token decay gradients add up to the per-channel one
    np.testing.assert_allclose(f[3].sum(axis=(0, 1)), e[3], rtol=1e-12, atol=1e-13)
