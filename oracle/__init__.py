"""TEST INFRASTRUCTURE ONLY: the CPU oracle of the RWKV-4 WKV recurrence.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
and imports nothing from it.

* ``forward``       -- fp64 max-trick recurrence in plain C (``wkv4_oracle.c``).
* ``decode``        -- repeated T=1 forward calls with the state carried in place.
* ``decode_slots``  -- one T=1 step per batch row on the state slot the row names
                       in a pool of states (gather, step, scatter).
* ``token_shift``   -- the token-shift mix of the current and the previous token.
* ``forward_gated`` / ``decode_gated`` -- the receptance gate of the time mix,
                       y = sigmoid(r) * wkv, applied to ``forward`` / ``decode``.
* ``combine_states`` -- one segment's state followed by another's (T split).
* ``brute``         -- the closed-form sums evaluated literally in 50-digit
                       arithmetic (``oracle/brute.py``), for tiny inputs.

The recurrence is the RWKV-4 WKV time mix whose fp32 per-channel numerator /
denominator / max state with the max-trick is described in "RWKV in a
self-built engine: a second non-attention paradigm (WKV/RNN)" (Methods table,
"Precision"; Reproducibility / Provenance, "Implementation").
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv4_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libwkv4_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, no fast-math) into oracle/_build."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            d = ctypes.POINTER(ctypes.c_double)
            lib.wkv4_oracle_forward.argtypes = [ctypes.c_int64] * 3 + [d] * 6 + [d, ctypes.c_int]
            lib.wkv4_oracle_forward.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor of any float dtype -> exact fp64 widening
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(k, v, w, u, state_in=None, *, want_y: bool = True, nthreads: int = 1):
    """fp64 forward over k, v [B, T, C]; w, u [C]; state_in [3, B, C] or None.

    Inputs are widened exactly to fp64 from whatever dtype they arrive in.
    Returns (y [B,T,C] or None, state_out [3,B,C]) as fp64 numpy arrays.
    """
    k, v, w, u, s_in = _f64(k), _f64(v), _f64(w), _f64(u), _f64(state_in)
    B, T, C = k.shape
    assert v.shape == (B, T, C) and w.shape == (C,) and u.shape == (C,)
    if s_in is not None:
        assert s_in.shape == (3, B, C)
    y = np.empty((B, T, C), dtype=np.float64) if want_y else None
    s_out = np.empty((3, B, C), dtype=np.float64)
    rc = _load().wkv4_oracle_forward(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s_in),
                                     _ptr(y), _ptr(s_out), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"wkv4_oracle_forward failed ({rc})")
    return y, s_out


def decode(k, v, w, u, state):
    """One T=1 step over k, v [B, C]: returns (y [B,C], new state [3,B,C])."""
    k, v = _f64(k), _f64(v)
    y, s = forward(k[:, None, :], v[:, None, :], w, u, state)
    return y[:, 0, :], s


def decode_slots(k, v, w, u, pool, slot_ids):
    """One T=1 step for each batch row b on pool row slot_ids[b].

    The RNN state as a first-class object the caller keeps per conversation
    ("An RNN that claims to match transformers, now in chatbot form", sections
    "The interesting bit" and "Caveats"), for many conversations at once:
    k, v [B, C]; pool [3, S, C]; slot_ids [B] integers.  Row b gathers its
    state from pool[:, slot_ids[b], :], takes the step of ``decode`` and
    scatters the new state back; a row whose id is outside [0, S) is skipped
    (its y row is NaN, the pool is not touched).  Returns (y [B, C], new pool
    [3, S, C], number of skipped rows) as fp64 numpy arrays.
    """
    k, v = _f64(k), _f64(v)
    pool = _f64(pool).copy()
    ids = np.asarray(slot_ids.detach().cpu() if hasattr(slot_ids, "detach") else slot_ids,
                     dtype=np.int64)
    B, C = k.shape
    S = pool.shape[1]
    assert pool.shape == (3, S, C) and ids.shape == (B,)
    y = np.full((B, C), np.nan)
    skipped = 0
    for b in range(B):
        s = int(ids[b])
        if s < 0 or s >= S:
            skipped += 1
            continue
        yb, sb = decode(k[b:b + 1], v[b:b + 1], w, u, pool[:, s:s + 1, :])
        y[b] = yb[0]
        pool[:, s, :] = sb[:, 0, :]
    return y, pool, skipped


def token_shift(x, x_prev, mixes):
    """Token shift of the time mix: each output mixes the current token with
    the previous one ("RWKV in a self-built engine: a second non-attention
    paradigm (WKV/RNN)", Reproducibility / Provenance, "Implementation":
    token-shift, "mix current and previous token"), read as
        out[b, t, c] = m[c] x[b, t, c] + (1 - m[c]) x[b, t - 1, c],
    x[b, -1, c] = x_prev[b, c] (zeros when x_prev is None), one output per mix
    vector in ``mixes``.  x [B, T, C]; returns (list of outputs [B, T, C],
    x_last [B, C]) in fp64.
    """
    x = _f64(x)
    B, T, C = x.shape
    prev = np.zeros((B, C)) if x_prev is None else _f64(x_prev)
    shifted = np.concatenate([prev[:, None, :], x[:, :-1, :]], axis=1)  # x[b, t - 1]
    outs = []
    for m in mixes:
        m = _f64(m)
        outs.append(m * x + (1.0 - m) * shifted)
    x_last = x[:, -1, :] if T > 0 else prev
    return outs, x_last


def sigmoid(r):
    """The logistic function 1 / (1 + e^{-r}) in fp64, elementwise (0 for r
    below about -709, where e^{-r} overflows, and 1 above about 37)."""
    r = _f64(r)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-r))


def forward_gated(k, v, r, w, u, state_in=None, *, nthreads: int = 1):
    """The WKV forward with the receptance gate of the time mix applied to its
    output: y = sigmoid(r) * wkv elementwise, r [B, T, C] ("RWKV in a
    self-built engine: a second non-attention paradigm (WKV/RNN)", abstract
    and Reproducibility / Provenance, "Implementation": time-mix gating;
    "RWKV-4 14B", "Every architecture field": the time mix's receptance
    matrix).  The pages name the gate and the receptance but not the gate's
    function; it is read as the logistic sigmoid.  The state does not depend
    on r.  Returns (y [B, T, C], state_out [3, B, C]) in fp64.
    """
    y, s = forward(k, v, w, u, state_in, nthreads=nthreads)
    return y * sigmoid(r), s


def decode_gated(k, v, r, w, u, state):
    """One T=1 step over k, v, r [B, C] with the receptance gate on its output:
    returns (sigmoid(r) * wkv [B, C], new state [3, B, C])."""
    y, s = decode(k, v, w, u, state)
    return y * sigmoid(r), s


def combine_states(x, y, n, w):
    """State x followed by a segment of n steps whose state from the empty
    state is y (both [3, B, C] planes num, den, max in natural units; n an
    int; w [C]): the state after both, X's numerator and denominator decayed
    by e^{n w}:  A = e^{n w} A_x + A_y,  D = e^{n w} D_x + D_y,  returned as a
    (num, den, max) triple with the max-trick (max = max(p_x + n w, p_y)).
    The state carried across a split of T ("An RNN that claims to match
    transformers, now in chatbot form", "The interesting bit": the state is
    the whole history).  fp64.
    """
    x, y, w = _f64(x), _f64(y), _f64(w)
    px = x[2] + n * w
    p = np.maximum(px, y[2])
    ex, ey = np.exp(px - p), np.exp(y[2] - p)
    return np.stack([ex * x[0] + ey * y[0], ex * x[1] + ey * y[1], p])


def empty_state(B: int, C: int) -> np.ndarray:
    s = np.zeros((3, B, C), dtype=np.float64)
    s[2] = -1e38
    return s
