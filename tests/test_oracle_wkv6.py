"""Pins for the fp64 Finch / RWKV-6 WKV oracle (the "Finch" section of the
Eagle/Finch summary page: the Eagle update s' = diag(w) s + k^T v with a decay
that depends on the token).  Each pin checks it against something other than
the recurrence itself: the Eagle oracle (pinned on its own) when the decay does
not move, hand-derived closed forms for the position of each token's decay,
a decay-zero token that must erase the past, the explicit sum over past tokens
with the decay products formed term by term, and split-sequence resume."""
import numpy as np
import pytest

import oracle
import wkv_inputs as wi


def _problem(B, T, H, N, seed, omega_range=(-6.0, 0.0), jitter=0.5):
    p = wi.wkv6_problem(B, T, H, N, seed, omega_range=omega_range, omega_jitter=jitter)
    return {k: v.double().numpy() for k, v in p.items()}


def test_constant_decay_is_eagle():
    # omega_t equal at every token: the Eagle recurrence with that omega.
    B, T, H, N = 2, 30, 2, 8
    p = wi.wkv5_problem(B, T, H, N, 11)
    p = {k: v.double().numpy() for k, v in p.items()}
    om_t = np.broadcast_to(p["omega"][None, None], (B, T, H, N)).copy()
    y6, s6 = oracle.wkv6_forward(p["r"], p["k"], p["v"], om_t, p["u"], return_state=True)
    y5, s5 = oracle.wkv5_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    np.testing.assert_allclose(y6, y5, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s6, s5, rtol=1e-13, atol=1e-15)


def test_three_tokens_decay_positions():
    # One channel, one value column: s after token 0 is k0 v0; token 1 multiplies
    # it by w1 and adds k1 v1; token 2 reads it.  So y2 = r2 (w1 k0 v0 + k1 v1 +
    # u k2 v2), and the final state is w2 w1 k0 v0 + w2 k1 v1 + k2 v2: w0 never
    # matters without an initial state.
    r = np.array([0.3, -0.7, 1.1]).reshape(1, 3, 1, 1)
    k = np.array([0.9, 0.4, -0.6]).reshape(1, 3, 1, 1)
    v = np.array([1.5, -2.0, 0.25]).reshape(1, 3, 1, 1)
    wv = np.array([0.2, 0.6, 0.8])
    omega = np.log(-np.log(wv)).reshape(1, 3, 1, 1)
    u = np.array([[0.5]])
    y, s = oracle.wkv6_forward(r, k, v, omega, u, return_state=True)
    r0, r1, r2 = r.ravel(); k0, k1, k2 = k.ravel(); v0, v1, v2 = v.ravel(); w0, w1, w2 = wv
    assert y[0, 0, 0, 0] == pytest.approx(r0 * 0.5 * k0 * v0, rel=1e-14)
    assert y[0, 1, 0, 0] == pytest.approx(r1 * (k0 * v0 + 0.5 * k1 * v1), rel=1e-14)
    assert y[0, 2, 0, 0] == pytest.approx(r2 * (w1 * k0 * v0 + k1 * v1 + 0.5 * k2 * v2), rel=1e-14)
    assert s[0, 0, 0, 0] == pytest.approx(w2 * w1 * k0 * v0 + w2 * k1 * v1 + k2 * v2, rel=1e-14)
    # with an initial state every token's decay applies to it, in order
    s0 = np.array([3.0]).reshape(1, 1, 1, 1)
    y, s = oracle.wkv6_forward(r, k, v, omega, u, s_in=s0, return_state=True)
    assert y[0, 0, 0, 0] == pytest.approx(r0 * (3.0 + 0.5 * k0 * v0), rel=1e-14)
    assert y[0, 2, 0, 0] == pytest.approx(r2 * (w1 * w0 * 3.0 + w1 * k0 * v0 + k1 * v1 + 0.5 * k2 * v2),
                                          rel=1e-14)


def test_zero_decay_token_erases_the_past():
    # omega = 8 at token m in every channel: w_m = exp(-e^8) underflows to 0, so
    # the state after m holds only k_m^T v_m and every later output equals that
    # of the same tokens started at m from a zero state.
    B, T, H, N, m = 2, 25, 2, 8, 9
    p = _problem(B, T, H, N, 12)
    om = p["omega"].copy()
    om[:, m] = 8.0
    y, s = oracle.wkv6_forward(p["r"], p["k"], p["v"], om, p["u"], return_state=True)
    sl = slice(m, T)
    y_tail, s_tail = oracle.wkv6_forward(p["r"][:, sl], p["k"][:, sl], p["v"][:, sl], om[:, sl], p["u"],
                                         return_state=True)
    np.testing.assert_allclose(y[:, m + 1:], y_tail[:, 1:], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s, s_tail, rtol=1e-13, atol=1e-15)
    assert not np.allclose(y[:, m], y_tail[:, 0])   # token m itself still reads the old state


def test_no_decay_unit_bonus_is_causal_linear_attention():
    # omega_t = -inf gives w_t = 1 at every token; with u = 1 the output is tril(r k^T) v.
    B, T, H, N = 1, 20, 2, 8
    p = _problem(B, T, H, N, 13)
    om = np.full((B, T, H, N), -np.inf)
    y = oracle.wkv6_forward(p["r"], p["k"], p["v"], om, np.ones((H, N)))
    for h in range(H):
        r, k, v = p["r"][0, :, h], p["k"][0, :, h], p["v"][0, :, h]
        np.testing.assert_allclose(y[0, :, h], np.tril(r @ k.T) @ v, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("omega_range", [(-6.0, 0.0), (-1.0, 2.0)])
def test_recurrence_equals_sum_over_past_tokens(omega_range):
    p = _problem(2, 14, 2, 8, 14, omega_range=omega_range, jitter=1.0)
    y_rec = oracle.wkv6_forward(p["r"], p["k"], p["v"], p["omega"], p["u"])
    y_sum = oracle.wkv6_forward_bruteforce(p["r"], p["k"], p["v"], p["omega"], p["u"])
    np.testing.assert_allclose(y_rec, y_sum, rtol=1e-11, atol=1e-14)


def test_split_sequence_resume():
    p = _problem(1, 40, 2, 16, 15)
    y_full, s_full = oracle.wkv6_forward(p["r"], p["k"], p["v"], p["omega"], p["u"], return_state=True)
    a, b = slice(0, 23), slice(23, 40)
    y1, s1 = oracle.wkv6_forward(p["r"][:, a], p["k"][:, a], p["v"][:, a], p["omega"][:, a], p["u"],
                                 return_state=True)
    y2, s2 = oracle.wkv6_forward(p["r"][:, b], p["k"][:, b], p["v"][:, b], p["omega"][:, b], p["u"],
                                 s_in=s1, return_state=True)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=1), y_full)
    np.testing.assert_array_equal(s2, s_full)


def test_planted_decay_offset_is_caught():
    # The pins above must reject a plausible indexing slip: decaying the state
    # with the NEXT token's w (w_{t+1} instead of w_t) is checked here against
    # the closed form of test_three_tokens_decay_positions.
    r = np.array([0.3, -0.7, 1.1]).reshape(1, 3, 1, 1)
    k = np.array([0.9, 0.4, -0.6]).reshape(1, 3, 1, 1)
    v = np.array([1.5, -2.0, 0.25]).reshape(1, 3, 1, 1)
    wv = np.array([0.2, 0.6, 0.8])
    shifted = np.roll(wv, -1)          # token t decays with w_{t+1}
    omega = np.log(-np.log(shifted)).reshape(1, 3, 1, 1)
    y = oracle.wkv6_forward(r, k, v, omega, np.array([[0.5]]))
    r2, k0, k1, k2, v0, v1, v2 = 1.1, 0.9, 0.4, -0.6, 1.5, -2.0, 0.25
    right = r2 * (wv[1] * k0 * v0 + k1 * v1 + 0.5 * k2 * v2)
    assert abs(y[0, 2, 0, 0] - right) > 1e-3
