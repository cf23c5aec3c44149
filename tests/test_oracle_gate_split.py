"""Pins of the oracle's receptance gate (forward_gated, decode_gated) and of its
state combine for a split of T (combine_states), against things other than
themselves:

* the gate: the logistic function against scipy's expit; its exact values at
  r = 0 (one half) and its limits at large |r|; the 50-digit closed form of
  the WKV sums times a 50-digit sigmoid; the state, which the gate must not
  touch; the decode step equal to one step of the gated forward;
* the combine: one call over T equals the first part's state combined with
  the second part's state from the empty state (checked against the 50-digit
  closed form of the whole sequence); the empty state is its identity; it is
  associative;
* planted mistakes in copies of both must fail these pins.
"""

import mpmath
import numpy as np
import pytest
import scipy.special

import oracle
from oracle import brute


def _inputs(seed, B=2, T=6, C=4, state=True):
    rng = np.random.default_rng(2000 + seed)
    k = rng.normal(0.0, 2.0, size=(B, T, C))
    v = rng.normal(0.0, 1.0, size=(B, T, C))
    r = rng.normal(0.0, 3.0, size=(B, T, C))
    k[0, min(1, T - 1), 2] = 30.0
    w = -np.exp(np.array([1.5, 0.0, -3.0, -8.0])[:C])
    u = np.array([-2.0, 0.5, 3.0, -0.2])[:C]
    s = None
    if state:
        s = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 2.0, size=(B, C)),
                      rng.uniform(-2.0, 2.0, size=(B, C))])
    return k, v, r, w, u, s


# ------------------------------------------------------------------ the gate

def test_sigmoid_matches_scipy_expit():
    r = np.concatenate([np.linspace(-50, 50, 2001), [-745.0, -709.0, -37.0, 37.0, 709.0, 1e-300]])
    got = oracle.sigmoid(r)
    ref = scipy.special.expit(r)
    np.testing.assert_allclose(got, ref, rtol=4e-16, atol=0.0)
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    assert oracle.sigmoid(np.array([-800.0]))[0] == 0.0
    assert oracle.sigmoid(np.array([800.0]))[0] == 1.0


def _gate_pins_hold(gated, seed=0):
    """Pins of a gated forward `gated(k, v, r, w, u, s) -> (y, state)`; True
    when every one holds."""
    k, v, r, w, u, s = _inputs(seed)
    y, st = oracle.forward(k, v, w, u, s)
    ok = True
    # r = 0: exactly half of wkv
    yg, sg = gated(k, v, np.zeros_like(r), w, u, s)
    ok &= bool(np.array_equal(yg, 0.5 * y))
    # r = +40: the gate is 1 to the last bit of fp64
    yg, _ = gated(k, v, np.full_like(r, 40.0), w, u, s)
    ok &= bool(np.array_equal(yg, y))
    # r = -40: the gate is e^-40 / (1 + e^-40)
    yg, _ = gated(k, v, np.full_like(r, -40.0), w, u, s)
    ok &= bool(np.allclose(yg, y * (np.exp(-40.0) / (1.0 + np.exp(-40.0))), rtol=1e-15, atol=0))
    # the state does not depend on r
    _, sg = gated(k, v, r, w, u, s)
    ok &= bool(np.array_equal(sg, st))
    # random r against the 50-digit closed form times a 50-digit sigmoid
    yg, _ = gated(k, v, r, w, u, s)
    yb, _, _ = brute.closed_form(k, v, w, u, s)
    B, T, C = k.shape
    for b in range(B):
        for t in range(T):
            for c in range(C):
                rr = mpmath.mpf(float(r[b, t, c]))
                ref = yb[b][t][c] / (1 + mpmath.exp(-rr))
                scale = max(abs(float(ref)), float(np.max(np.abs(v[b, : t + 1, c]))) * 1e-3)
                ok &= abs(yg[b, t, c] - float(ref)) <= 1e-12 * scale
    return ok


@pytest.mark.parametrize("seed", [0, 1])
def test_gated_forward_pins(seed):
    assert _gate_pins_hold(oracle.forward_gated, seed)


def test_gated_forward_without_state():
    k, v, r, w, u, _ = _inputs(5, state=False)
    yg, sg = oracle.forward_gated(k, v, r, w, u, None)
    yb, Ab, Db = brute.closed_form(k, v, w, u, None)
    for idx in np.ndindex(*k.shape):
        b, t, c = idx
        ref = yb[b][t][c] / (1 + mpmath.exp(-mpmath.mpf(float(r[idx]))))
        assert abs(yg[idx] - float(ref)) <= 1e-12 * max(1.0, abs(float(ref)))


def test_decode_gated_is_one_step_of_the_gated_forward():
    k, v, r, w, u, s = _inputs(3, T=1)
    y1, s1 = oracle.forward_gated(k, v, r, w, u, s)
    yd, sd = oracle.decode_gated(k[:, 0], v[:, 0], r[:, 0], w, u, s)
    assert np.array_equal(yd, y1[:, 0]) and np.array_equal(sd, s1)


def test_planted_gate_mistakes_fail_the_pins():
    def wrong_sign(k, v, r, w, u, s):          # sigmoid(-r)
        y, st = oracle.forward(k, v, w, u, s)
        return y * oracle.sigmoid(-r), st

    def tanh_gate(k, v, r, w, u, s):           # another squashing function
        y, st = oracle.forward(k, v, w, u, s)
        return y * np.tanh(r), st

    def ungated(k, v, r, w, u, s):             # gate left out
        return oracle.forward(k, v, w, u, s)

    def gate_on_k(k, v, r, w, u, s):           # gate taken from the wrong input
        y, st = oracle.forward(k, v, w, u, s)
        return y * oracle.sigmoid(k), st

    def gate_inside_state(k, v, r, w, u, s):   # gate applied to v before the recurrence
        return oracle.forward(k, v * oracle.sigmoid(r), w, u, s)

    for bad in (wrong_sign, tanh_gate, ungated, gate_on_k, gate_inside_state):
        assert not _gate_pins_hold(bad), bad.__name__


# --------------------------------------------------------- the state combine

def _split_pin_holds(combine, seed=0, split=3):
    """One call over T against the first `split` steps' state combined with
    the rest's state from the empty state, and that against the 50-digit
    closed form of the whole sequence."""
    k, v, _, w, u, s = _inputs(seed, T=7)
    _, s_all = oracle.forward(k, v, w, u, s)
    _, s1 = oracle.forward(k[:, :split], v[:, :split], w, u, s)
    _, s2 = oracle.forward(k[:, split:], v[:, split:], w, u, None)
    sc = combine(s1, s2, k.shape[1] - split, w)
    _, Ab, Db = brute.closed_form(k, v, w, u, s)
    ok = True
    B, _, C = k.shape
    for b in range(B):
        for c in range(C):
            e = mpmath.exp(mpmath.mpf(float(sc[2, b, c])))
            A = mpmath.mpf(float(sc[0, b, c])) * e
            D = mpmath.mpf(float(sc[1, b, c])) * e
            ok &= abs(D - Db[b][c]) <= 1e-12 * Db[b][c]
            ok &= abs(A - Ab[b][c]) <= 1e-12 * Db[b][c] * max(1.0, float(np.max(np.abs(v[b, :, c]))))
    # and the same numbers as the single call's own state (max-trick form)
    m = np.maximum(sc[2], s_all[2])
    ok &= bool(np.allclose(sc[1] * np.exp(sc[2] - m), s_all[1] * np.exp(s_all[2] - m), rtol=1e-13))
    return ok


@pytest.mark.parametrize("split", [1, 3, 6])
@pytest.mark.parametrize("seed", [0, 1])
def test_combine_equals_one_call_over_the_split(seed, split):
    assert _split_pin_holds(oracle.combine_states, seed, split)


def test_combine_identity_and_decay():
    rng = np.random.default_rng(9)
    B, C = 3, 4
    w = -np.exp(rng.uniform(-6, 1, size=C))
    x = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 2, size=(B, C)),
                  rng.uniform(-2, 2, size=(B, C))])
    e = oracle.empty_state(B, C)
    # empty, then y: y itself
    assert np.array_equal(oracle.combine_states(e, x, 5, w), x)
    # x, then an empty segment of n steps: x decayed by e^{n w} (in the max)
    xd = oracle.combine_states(x, e, 5, w)
    assert np.array_equal(xd[0], x[0]) and np.array_equal(xd[1], x[1])
    np.testing.assert_allclose(xd[2], x[2] + 5 * w, rtol=0, atol=1e-15)


def test_combine_is_associative():
    k, v, _, w, u, s = _inputs(4, T=9)
    parts = [(0, 2), (2, 6), (6, 9)]
    st = [oracle.forward(k[:, a:b_], v[:, a:b_], w, u, None)[1] for a, b_ in parts]
    left = oracle.combine_states(oracle.combine_states(st[0], st[1], 4, w), st[2], 3, w)
    right = oracle.combine_states(st[0], oracle.combine_states(st[1], st[2], 3, w), 7, w)
    m = np.maximum(left[2], right[2])
    for i in (0, 1):
        np.testing.assert_allclose(left[i] * np.exp(left[2] - m), right[i] * np.exp(right[2] - m),
                                   rtol=1e-13, atol=1e-300)


def test_planted_combine_mistakes_fail_the_pin():
    def decay_second(x, y, n, w):   # decays the later segment instead of the earlier one
        return oracle.combine_states(y, x, n, w)

    def off_by_one(x, y, n, w):     # n - 1 steps of decay
        return oracle.combine_states(x, y, n - 1, w)

    def no_decay(x, y, n, w):       # the earlier state joined undecayed
        return oracle.combine_states(x, y, 0, w)

    for bad in (decay_second, off_by_one, no_decay):
        assert not _split_pin_holds(bad), bad.__name__
