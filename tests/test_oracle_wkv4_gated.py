"""Pins for the fp64 receptance-gated WKV-4 oracle (P1 (2): the time-mixing
output is W_o (sigmoid(r_t) * WKV_t); the operator computes the gated part).
Each pin checks it against something other than its own formula: the gate's
fixed points (fully open, half open), the symmetry sigmoid(-x) = 1 - sigmoid(x),
and central finite differences of L = sum(go * o) for every input."""
import numpy as np
import pytest

import oracle
import wkv_inputs as wi


def _problem(B, T, C, seed):
    p = wi.wkv4_problem(B, T, C, seed, with_gy=True, gated=True)
    return {k: v.double().numpy() for k, v in p.items()}


def test_open_gate_is_the_plain_operator():
    # r = 40: sigmoid(r) = 1 - 4e-18, so the gated output and the gradients of k, v, w, u are the
    # plain operator's with gy = go, and gr vanishes
    p = _problem(2, 30, 4, 21)
    r = np.full_like(p["k"], 40.0)
    o = oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], r)
    y = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    np.testing.assert_allclose(o, y, rtol=1e-15, atol=1e-15)
    gk, gv, gr, gw, gu = oracle.wkv4_gated_backward(p["w"], p["u"], p["k"], p["v"], r, p["go"])
    ref = oracle.wkv4_backward(p["w"], p["u"], p["k"], p["v"], p["go"])
    for got, want in zip((gk, gv, gw, gu), ref):
        np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    assert np.max(np.abs(gr)) < 1e-15


def test_half_open_gate_and_symmetry():
    p = _problem(2, 25, 3, 22)
    y = oracle.wkv4_forward(p["w"], p["u"], p["k"], p["v"])
    o0 = oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], np.zeros_like(p["k"]))
    np.testing.assert_allclose(o0, 0.5 * y, rtol=1e-15, atol=0)
    o_pos = oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], p["r"])
    o_neg = oracle.wkv4_gated_forward(p["w"], p["u"], p["k"], p["v"], -p["r"])
    np.testing.assert_allclose(o_pos + o_neg, y, rtol=1e-13, atol=1e-15)
    # gr at r = 0 is go * y * 1/4
    gr0 = oracle.wkv4_gated_backward(p["w"], p["u"], p["k"], p["v"], np.zeros_like(p["k"]), p["go"])[2]
    np.testing.assert_allclose(gr0, 0.25 * p["go"] * y, rtol=1e-15, atol=0)


@pytest.mark.parametrize("with_state", [False, True])
def test_gradients_match_finite_differences(with_state):
    B, T, C, h = 1, 12, 3, 1e-6
    p = _problem(B, T, C, 23)
    s0 = None
    if with_state:
        _, s0 = oracle.wkv4_forward(p["w"], p["u"], p["k"][:, :5], p["v"][:, :5], return_state=True)

    def loss(q):
        return float(np.sum(q["go"] * oracle.wkv4_gated_forward(q["w"], q["u"], q["k"], q["v"], q["r"],
                                                                 state_in=s0)))

    gk, gv, gr, gw, gu = oracle.wkv4_gated_backward(p["w"], p["u"], p["k"], p["v"], p["r"], p["go"],
                                                    state_in=s0)
    for name, grad in (("k", gk), ("v", gv), ("r", gr), ("w", gw), ("u", gu)):
        num = np.zeros_like(p[name])
        for idx in np.ndindex(p[name].shape):
            qp = {k: v.copy() for k, v in p.items()}
            qm = {k: v.copy() for k, v in p.items()}
            qp[name][idx] += h
            qm[name][idx] -= h
            num[idx] = (loss(qp) - loss(qm)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)
