"""Pins of the fp64 oracle against things other than itself.

* the closed-form sums in 50-digit arithmetic (brute force, tiny inputs);
* invariants that hold for any correct implementation (constant v, convex
  hull of the prefix, T=1, chaining two calls equals one call);
* limits that reduce to a textbook softmax (w -> -inf and w = 0);
* the linear-domain recurrence without rescaling where it cannot overflow,
  and its overflow where the max-trick is needed;
* planted mistakes in a copy of the oracle's C source must fail these pins.
"""

import ctypes
import os
import subprocess

import mpmath
import numpy as np
import pytest
import scipy.special

import oracle
from oracle import brute

ORACLE_SRC = os.path.join(os.path.dirname(oracle.__file__), "wkv4_oracle.c")


def _tiny_inputs(seed, B=2, T=7, C=4, state=True, spikes=True):
    rng = np.random.default_rng(1000 + seed)
    k = rng.normal(0.0, 2.0, size=(B, T, C))
    v = rng.normal(0.0, 1.0, size=(B, T, C))
    if spikes:
        k[0, 2, 1] = 30.0
        k[B - 1, T - 1, 0] = 30.0
    # decays from very fast to very slow, as -exp(time_decay) with td in [-8, 2]
    w = -np.exp(np.array([2.0, 0.0, -3.0, -8.0])[:C])
    u = np.array([-3.0, 0.5, 3.0, -0.2])[:C]
    s = None
    if state:
        s = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 2.0, size=(B, C)),
                      rng.uniform(-2.0, 2.0, size=(B, C))])
    return k, v, w, u, s


def _check_against_closed_form(fwd, k, v, w, u, s, rel=1e-12):
    """fwd(k, v, w, u, s) -> (y, state_out); compares with the literal sums."""
    y, s_out = fwd(k, v, w, u, s)
    yb, Ab, Db = brute.closed_form(k, v, w, u, s)
    B, T, C = k.shape
    for b in range(B):
        for c in range(C):
            for t in range(T):
                ref = yb[b][t][c]
                scale = max(abs(float(ref)), float(np.max(np.abs(v[b, : t + 1, c]))))
                assert abs(y[b, t, c] - float(ref)) <= rel * scale, (b, t, c, y[b, t, c], ref)
            # state: compare A = a e^p and D = b e^p relative to D
            e = mpmath.exp(mpmath.mpf(float(s_out[2, b, c])))
            A = mpmath.mpf(float(s_out[0, b, c])) * e
            D = mpmath.mpf(float(s_out[1, b, c])) * e
            assert abs(D - Db[b][c]) <= rel * Db[b][c], (b, c)
            assert abs(A - Ab[b][c]) <= rel * Db[b][c] * max(1.0, float(np.max(np.abs(v[b, :, c])))), (b, c)


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("state", [False, True])
def test_closed_form_brute_force(seed, state):
    k, v, w, u, s = _tiny_inputs(seed, state=state)
    _check_against_closed_form(oracle.forward, k, v, w, u, s)


def test_closed_form_extreme_decays_and_bonus():
    k, v, _, _, s = _tiny_inputs(7, T=8)
    w = np.array([-7.389, -3.4e-4, -1e-9, -20.0])
    u = np.array([3.0, -3.0, 0.0, 10.0])
    _check_against_closed_form(oracle.forward, k, v, w, u, s)


def test_constant_v_gives_constant_output():
    rng = np.random.default_rng(3)
    B, T, C = 2, 50, 5
    k = rng.normal(0, 2, size=(B, T, C))
    v = np.full((B, T, C), 0.7318)
    w = -np.exp(rng.uniform(-6, 1, size=C))
    u = rng.uniform(-1, 1, size=C)
    y, _ = oracle.forward(k, v, w, u, None)
    np.testing.assert_allclose(y, 0.7318, rtol=1e-14, atol=0)


def test_output_in_convex_hull_of_prefix():
    rng = np.random.default_rng(4)
    B, T, C = 3, 64, 6
    k = rng.normal(0, 2, size=(B, T, C))
    k[1, 10, 2] = 30.0
    v = rng.normal(0, 1, size=(B, T, C))
    w = -np.exp(rng.uniform(-8, 2, size=C))
    u = rng.uniform(-3, 3, size=C)
    y, _ = oracle.forward(k, v, w, u, None)
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    slack = 1e-13
    assert np.all(y >= lo - slack) and np.all(y <= hi + slack)


def test_single_step_empty_state_returns_v():
    rng = np.random.default_rng(5)
    k = rng.normal(0, 2, size=(4, 1, 9))
    v = rng.normal(0, 1, size=(4, 1, 9))
    w = -np.exp(rng.uniform(-6, 1, size=9))
    u = rng.uniform(-1, 1, size=9)
    y, s = oracle.forward(k, v, w, u, None)
    np.testing.assert_allclose(y, v, rtol=1e-15, atol=0)
    # after one token the state is (v, 1, k): A = e^k v, D = e^k
    np.testing.assert_allclose(s[0] * np.exp(s[2]), np.exp(k[:, 0]) * v[:, 0], rtol=1e-14)
    np.testing.assert_allclose(s[1] * np.exp(s[2]), np.exp(k[:, 0]), rtol=1e-14)


@pytest.mark.parametrize("split", [1, 17, 63])
def test_two_calls_with_carried_state_equal_one_call(split):
    rng = np.random.default_rng(6)
    B, T, C = 2, 64, 5
    k = rng.normal(0, 2, size=(B, T, C))
    k[0, 5, 1] = 30.0
    v = rng.normal(0, 1, size=(B, T, C))
    w = -np.exp(rng.uniform(-8, 2, size=C))
    u = rng.uniform(-3, 3, size=C)
    s0 = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 2, size=(B, C)),
                   rng.uniform(-2, 2, size=(B, C))])
    y, s = oracle.forward(k, v, w, u, s0)
    y1, s1 = oracle.forward(k[:, :split], v[:, :split], w, u, s0)
    y2, s2 = oracle.forward(k[:, split:], v[:, split:], w, u, s1)
    # the recurrence is sequential, so carrying the fp64 state is exact
    assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
    assert np.array_equal(s2, s)


def test_decode_steps_equal_forward():
    rng = np.random.default_rng(8)
    B, T, C = 3, 12, 4
    k = rng.normal(0, 2, size=(B, T, C))
    v = rng.normal(0, 1, size=(B, T, C))
    w = -np.exp(rng.uniform(-6, 1, size=C))
    u = rng.uniform(-1, 1, size=C)
    y, s = oracle.forward(k, v, w, u, None)
    st = oracle.empty_state(B, C)
    for t in range(T):
        yt, st = oracle.decode(k[:, t], v[:, t], w, u, st)
        assert np.array_equal(yt, y[:, t])
    assert np.array_equal(st, s)


def test_fast_decay_limit_is_two_term_softmax():
    """w -> -inf: only the previous token survives the decay, so y_t is the
    softmax average of v_{t-1}, v_t with logits k_{t-1}, u + k_t."""
    rng = np.random.default_rng(9)
    B, T, C = 2, 20, 3
    k = rng.normal(0, 2, size=(B, T, C))
    v = rng.normal(0, 1, size=(B, T, C))
    w = np.full(C, -1e30)
    u = rng.uniform(-1, 1, size=C)
    y, _ = oracle.forward(k, v, w, u, None)
    for b in range(B):
        for c in range(C):
            assert y[b, 0, c] == pytest.approx(v[b, 0, c], rel=1e-15)
            for t in range(1, T):
                p = scipy.special.softmax([k[b, t - 1, c], u[c] + k[b, t, c]])
                ref = p[0] * v[b, t - 1, c] + p[1] * v[b, t, c]
                assert y[b, t, c] == pytest.approx(ref, rel=1e-12, abs=1e-14)


def test_no_decay_limit_is_cumulative_softmax():
    """w = 0: y_t is the softmax average of v_0..v_t with logits k_i (i < t)
    and u + k_t."""
    rng = np.random.default_rng(10)
    B, T, C = 2, 30, 3
    k = rng.normal(0, 2, size=(B, T, C))
    k[1, 3, 2] = 30.0
    v = rng.normal(0, 1, size=(B, T, C))
    w = np.zeros(C)
    u = rng.uniform(-1, 1, size=C)
    y, _ = oracle.forward(k, v, w, u, None)
    for b in range(B):
        for c in range(C):
            for t in range(T):
                logits = np.concatenate([k[b, :t, c], [u[c] + k[b, t, c]]])
                p = scipy.special.softmax(logits)
                assert y[b, t, c] == pytest.approx(np.dot(p, v[b, : t + 1, c]), rel=1e-12, abs=1e-14)


def test_matches_unscaled_recurrence_when_it_cannot_overflow():
    rng = np.random.default_rng(11)
    B, T, C = 2, 20, 4
    k = rng.normal(0, 1, size=(B, T, C))
    v = rng.normal(0, 1, size=(B, T, C))
    w = -np.exp(rng.uniform(-6, 1, size=C))
    u = rng.uniform(-1, 1, size=C)
    y, s = oracle.forward(k, v, w, u, None)
    A = np.zeros((B, C))
    D = np.zeros((B, C))
    for t in range(T):
        eb = np.exp(u + k[:, t])
        ref = (A + eb * v[:, t]) / (D + eb)
        np.testing.assert_allclose(y[:, t], ref, rtol=1e-13, atol=1e-15)
        A = np.exp(w) * A + np.exp(k[:, t]) * v[:, t]
        D = np.exp(w) * D + np.exp(k[:, t])
    np.testing.assert_allclose(s[0] * np.exp(s[2]), A, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(s[1] * np.exp(s[2]), D, rtol=1e-13)


def test_max_trick_survives_where_unscaled_overflows():
    B, T, C = 1, 6, 2
    k = np.zeros((B, T, C))
    k[0, 1, :] = 800.0  # e^800 overflows fp64
    k[0, 3, :] = 790.0
    v = np.arange(B * T * C, dtype=np.float64).reshape(B, T, C) / 7.0 - 0.5
    w = np.array([-0.5, -5.0])
    u = np.array([0.25, -1.0])
    with np.errstate(over="ignore", invalid="ignore"):
        assert not np.isfinite(np.exp(800.0) * v[0, 1, 0] / np.exp(800.0))
    y, s = oracle.forward(k, v, w, u, None)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(s))
    _check_against_closed_form(oracle.forward, k, v, w, u, None)


# ---------------------------------------------------------------------------
# planted mistakes: a copy of the oracle with one plausible bug must fail

MUTATIONS = {
    "dropped_bonus": ("const double q = fmax(p, u + kt);", "const double q = fmax(p, kt);",
                      "const double e_bonus = exp(u + kt - q);", "const double e_bonus = exp(kt - q);"),
    "wrong_decay_sign": ("const double q2 = fmax(p + w, kt);", "const double q2 = fmax(p - w, kt);",
                         "const double e_decay = exp(p + w - q2);", "const double e_decay = exp(p - w - q2);"),
    "state_in_ignored": ("if (j->state_in) {", "if (0) {"),
    "update_before_output": None,  # built below
    "kill_wkv": ("if (j->y) j->y[idx] = (e_state * a + e_bonus * vt) / (e_state * d + e_bonus);",
                 "if (j->y) j->y[idx] = vt;"),
    "den_without_state": ("(e_state * d + e_bonus)", "(e_bonus)"),
}


def _mutant_source(name):
    src = open(ORACLE_SRC).read()
    if name == "update_before_output":
        out_block = ("        /* output at step t */\n"
                     "        const double q = fmax(p, u + kt);\n"
                     "        const double e_state = exp(p - q);\n"
                     "        const double e_bonus = exp(u + kt - q);\n"
                     "        if (j->y) j->y[idx] = (e_state * a + e_bonus * vt) / (e_state * d + e_bonus);\n")
        upd_block = ("        /* state update */\n"
                     "        const double q2 = fmax(p + w, kt);\n"
                     "        const double e_decay = exp(p + w - q2);\n"
                     "        const double e_new = exp(kt - q2);\n"
                     "        a = e_decay * a + e_new * vt;\n"
                     "        d = e_decay * d + e_new;\n"
                     "        p = q2;\n")
        assert out_block + upd_block in src
        return src.replace(out_block + upd_block, upd_block + out_block)
    pairs = MUTATIONS[name]
    for old, new in zip(pairs[::2], pairs[1::2]):
        assert old in src, old
        src = src.replace(old, new)
    return src


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = tmp_path / "mutant.c"
    src.write_text(_mutant_source(name))
    lib_path = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o",
                           str(lib_path), str(src), "-lm"])
    lib = ctypes.CDLL(str(lib_path))
    dp = ctypes.POINTER(ctypes.c_double)
    lib.wkv4_oracle_forward.argtypes = [ctypes.c_int64] * 3 + [dp] * 6 + [dp, ctypes.c_int]

    def fwd(k, v, w, u, s):
        arrs = [np.ascontiguousarray(x, dtype=np.float64) if x is not None else None
                for x in (w, u, k, v, s)]
        B, T, C = k.shape
        y = np.empty((B, T, C))
        so = np.empty((3, B, C))
        ptrs = [a.ctypes.data_as(dp) if a is not None else None for a in arrs]
        lib.wkv4_oracle_forward(B, T, C, *ptrs, y.ctypes.data_as(dp), so.ctypes.data_as(dp), 1)
        return y, so

    k, v, w, u, s = _tiny_inputs(0, state=True)
    with pytest.raises(AssertionError):
        _check_against_closed_form(fwd, k, v, w, u, s)


def test_golden_closed_form_fixture():
    import json
    path = os.path.join(os.path.dirname(__file__), "golden", "closed_form_tiny.json")
    doc = json.load(open(path))
    k, v = np.array(doc["k"]), np.array(doc["v"])
    w, u = np.array(doc["w"]), np.array(doc["u"])
    for case in doc["cases"]:
        s = None if case["state_in"] is None else np.array(case["state_in"])
        y, so = oracle.forward(k, v, w, u, s)
        ref = np.array([[[float(x) for x in row] for row in yb] for yb in case["y"]])
        np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
        A = np.array([[float(x) for x in r] for r in case["A_out"]])
        D = np.array([[float(x) for x in r] for r in case["D_out"]])
        np.testing.assert_allclose(so[1] * np.exp(so[2]), D, rtol=1e-13)
        np.testing.assert_allclose(so[0] * np.exp(so[2]), A, rtol=1e-13, atol=1e-13 * np.max(D))


# ---- slot-indexed decode: gather the named pool row, take the step, scatter back

def test_slot_decode_matches_closed_form_on_the_named_rows():
    rng = np.random.default_rng(77)
    S, B, C = 5, 3, 4
    _, _, w, u, _ = _tiny_inputs(0, C=C)
    pool = np.stack([rng.normal(size=(S, C)), rng.uniform(0.5, 2.0, size=(S, C)),
                     rng.uniform(-2.0, 2.0, size=(S, C))])
    ids = np.array([4, 0, 2])
    k = rng.normal(0.0, 2.0, size=(B, C))
    v = rng.normal(size=(B, C))
    y, new_pool, skipped = oracle.decode_slots(k, v, w, u, pool, ids)
    assert skipped == 0
    gathered = pool[:, ids, :]
    yb, Ab, Db = brute.closed_form(k[:, None, :], v[:, None, :], w, u, gathered)
    for b in range(B):
        for c in range(C):
            ref = float(yb[b][0][c])
            assert abs(y[b, c] - ref) <= 1e-12 * max(abs(ref), abs(v[b, c])), (b, c)
            s = ids[b]
            e = mpmath.exp(mpmath.mpf(float(new_pool[2, s, c])))
            D = mpmath.mpf(float(new_pool[1, s, c])) * e
            A = mpmath.mpf(float(new_pool[0, s, c])) * e
            assert abs(D - Db[b][c]) <= 1e-12 * Db[b][c]
            assert abs(A - Ab[b][c]) <= 1e-12 * Db[b][c] * max(1.0, abs(v[b, c]))
    untouched = [s for s in range(S) if s not in ids]
    assert np.array_equal(new_pool[:, untouched, :], pool[:, untouched, :])


def test_slot_decode_permuted_ids_follow_their_rows():
    rng = np.random.default_rng(5)
    S = B = 9
    C = 4
    _, _, w, u, _ = _tiny_inputs(1, C=C)
    pool = np.stack([rng.normal(size=(S, C)), rng.uniform(0.5, 2.0, size=(S, C)),
                     rng.uniform(-2.0, 2.0, size=(S, C))])
    perm = rng.permutation(S)
    k = rng.normal(0.0, 2.0, size=(B, C))
    v = rng.normal(size=(B, C))
    y, new_pool, _ = oracle.decode_slots(k, v, w, u, pool, perm)
    # row b's result depends only on pool row perm[b] and is written back there
    y_ref, s_ref = oracle.decode(k, v, w, u, pool[:, perm, :])
    assert np.array_equal(y, y_ref)
    assert np.array_equal(new_pool[:, perm, :], s_ref)
    # the identity permutation is the plain decode
    y_id, s_id, _ = oracle.decode_slots(k, v, w, u, pool, np.arange(S))
    y_plain, s_plain = oracle.decode(k, v, w, u, pool)
    assert np.array_equal(y_id, y_plain) and np.array_equal(s_id, s_plain)


def test_slot_decode_skips_ids_outside_the_pool():
    rng = np.random.default_rng(9)
    S, C = 4, 4
    _, _, w, u, _ = _tiny_inputs(2, C=C)
    pool = np.stack([rng.normal(size=(S, C)), rng.uniform(0.5, 2.0, size=(S, C)),
                     rng.uniform(-2.0, 2.0, size=(S, C))])
    ids = np.array([1, -1, S, 3])
    k = rng.normal(size=(4, C))
    v = rng.normal(size=(4, C))
    y, new_pool, skipped = oracle.decode_slots(k, v, w, u, pool, ids)
    assert skipped == 2
    assert np.all(np.isnan(y[1])) and np.all(np.isnan(y[2]))
    assert np.all(np.isfinite(y[[0, 3]]))
    assert np.array_equal(new_pool[:, [0, 2], :], pool[:, [0, 2], :])
    assert not np.array_equal(new_pool[:, 1, :], pool[:, 1, :])


# ---- token shift: a per-channel mix of the current and the previous token

def _shift_inputs(seed, B=3, T=9, C=5):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(B, T, C)), rng.normal(size=(B, C))


def test_token_shift_special_mixes_select_a_token():
    x, xp = _shift_inputs(0)
    ones, zeros = np.ones(5), np.zeros(5)
    (cur, prev), last = oracle.token_shift(x, xp, [ones, zeros])
    assert np.array_equal(cur, x)                       # mix 1: the current token
    assert np.array_equal(prev[:, 0], xp)               # mix 0 at t = 0: the carried token
    assert np.array_equal(prev[:, 1:], x[:, :-1])       # mix 0 later: the previous token
    assert np.array_equal(last, x[:, -1])
    (first,), _ = oracle.token_shift(x, None, [zeros])
    assert np.array_equal(first[:, 0], np.zeros((3, 5)))  # a sequence start mixes with zeros


def test_token_shift_mixes_are_per_channel():
    x, xp = _shift_inputs(1)
    m = np.array([1.0, 0.0, 0.5, 0.25, 1.0])
    (out,), _ = oracle.token_shift(x, xp, [m])
    sh = np.concatenate([xp[:, None], x[:, :-1]], axis=1)
    assert np.array_equal(out[..., 0], x[..., 0]) and np.array_equal(out[..., 4], x[..., 4])
    assert np.array_equal(out[..., 1], sh[..., 1])
    assert np.allclose(out[..., 2], (x[..., 2] + sh[..., 2]) / 2, rtol=0, atol=1e-15)
    # a convex combination: between the two tokens
    lo, hi = np.minimum(x, sh), np.maximum(x, sh)
    assert np.all(out >= lo - 1e-15) and np.all(out <= hi + 1e-15)


@pytest.mark.parametrize("split", [1, 4, 8])
def test_token_shift_chained_calls_equal_one_call(split):
    x, xp = _shift_inputs(2)
    m = np.random.default_rng(3).uniform(size=5)
    (whole,), last = oracle.token_shift(x, xp, [m])
    (a,), mid = oracle.token_shift(x[:, :split], xp, [m])
    (b,), last2 = oracle.token_shift(x[:, split:], mid, [m])
    assert np.array_equal(np.concatenate([a, b], axis=1), whole)
    assert np.array_equal(last, last2)
