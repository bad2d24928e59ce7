"""Pins for the fp64 Eagle / RWKV-5 WKV oracle (the "Eagle" section of the
Eagle/Finch summary page: s' = diag(w) s + k^T v, wkv' = s + diag(u) k^T v,
w = exp(-exp(omega))), each against something other than the recurrence
itself: the one-token closed form, causal linear attention as a masked
matrix product, the fast-decay limit, the explicit sum over past tokens, and
split-sequence resume."""
import numpy as np
import pytest

import oracle
import wkv_inputs as wi


def _problem(B, T, H, N, seed, omega_range=(-6.0, 0.0)):
    p = wi.wkv5_problem(B, T, H, N, seed, omega_range=omega_range)
    return {k: v.double().numpy() for k, v in p.items()}


def test_single_token_closed_form():
    p = _problem(2, 1, 3, 16, 1)
    y, s = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    r, k, v = p["r"][:, 0], p["k"][:, 0], p["v"][:, 0]  # [B, H, N]
    bonus = np.sum(r * p["u"][None] * k, axis=-1, keepdims=True)
    np.testing.assert_allclose(y[:, 0], bonus * v, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s, k[..., :, None] * v[..., None, :], rtol=1e-15, atol=0)


def test_no_decay_unit_bonus_is_causal_linear_attention():
    # omega = -inf gives w = 1; with u = 1 the output is tril(r k^T) v.
    B, T, H, N = 1, 24, 2, 8
    p = _problem(B, T, H, N, 2)
    omega = np.full((H, N), -np.inf)
    u = np.ones((H, N))
    y = oracle.wkv5_forward(p["r"], p["k"], p["v"], omega, u)
    for h in range(H):
        r, k, v = p["r"][0, :, h], p["k"][0, :, h], p["v"][0, :, h]
        expect = np.tril(r @ k.T) @ v
        np.testing.assert_allclose(y[0, :, h], expect, rtol=1e-12, atol=1e-14)


def test_fast_decay_keeps_previous_token_only():
    # omega = 5: w = exp(-e^5) ~ e^-148, so only the lag-0 past token survives.
    B, T, H, N = 1, 20, 2, 8
    p = _problem(B, T, H, N, 3)
    omega = np.full((H, N), 5.0)
    y = oracle.wkv5_forward(p["r"], p["k"], p["v"], omega, p["u"])
    r, k, v, u = p["r"][0], p["k"][0], p["v"][0], p["u"]
    cur = np.sum(r * u[None] * k, axis=-1, keepdims=True) * v
    prev = np.zeros_like(cur)
    prev[1:] = np.sum(r[1:] * k[:-1], axis=-1, keepdims=True) * v[:-1]
    np.testing.assert_allclose(y[0], cur + prev, rtol=1e-12, atol=1e-14)


def test_recurrence_equals_sum_over_past_tokens():
    p = _problem(2, 20, 2, 8, 4)
    y_rec = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"])
    y_sum = oracle.wkv5_forward_bruteforce(p["r"], p["k"], p["v"], p["omega"], p["u"])
    np.testing.assert_allclose(y_rec, y_sum, rtol=1e-11, atol=1e-14)


def test_state_layout_rows_are_keys():
    # diag(w) must scale the key (row) index: give keys along one axis only and
    # check that the decay of that row, not of a column, is applied.
    B, T, H, N = 1, 2, 1, 4
    r = np.zeros((B, T, H, N)); k = np.zeros_like(r); v = np.zeros_like(r)
    k[0, 0, 0, 1] = 1.0          # key index 1
    v[0, 0, 0, 2] = 1.0          # value index 2
    r[0, 1, 0, 1] = 1.0          # read key row 1 at t = 1
    omega = np.log(-np.log(np.array([[0.9, 0.5, 0.7, 0.3]])))   # w = (.9,.5,.7,.3)
    y, s = oracle.wkv5_forward(r, k, v, omega, np.zeros((H, N)), return_state=True)
    assert y[0, 1, 0, 2] == pytest.approx(1.0)                  # lag 0: weight w^0
    assert s[0, 0, 1, 2] == pytest.approx(0.5)                  # decayed by w_1 = .5
    assert np.count_nonzero(s) == 1


def test_split_sequence_resume():
    p = _problem(1, 40, 2, 16, 5)
    y_full, s_full = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"],
                                         return_state=True)
    sl = slice(0, 17), slice(17, 40)
    y1, s1 = oracle.wkv5_forward(p["r"][:, sl[0]], p["k"][:, sl[0]], p["v"][:, sl[0]],
                                 p["omega"], p["u"], return_state=True)
    y2, s2 = oracle.wkv5_forward(p["r"][:, sl[1]], p["k"][:, sl[1]], p["v"][:, sl[1]],
                                 p["omega"], p["u"], s_in=s1, return_state=True)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=1), y_full)
    np.testing.assert_array_equal(s2, s_full)
