"""Parity gates between the CUDA path and the fp64 oracle.

y, fp32 I/O:       max |y - y_ref| <= 2e-5 * max|v|   (max over the call's v)
y, fp16/bf16 I/O:  |y - y_ref| <= 2 ulp_dtype(|y_ref|) + 1e-3 |y_ref|
                                  + (K_ARITH + calls) 2^-24 y_abs,   elementwise.
                   The first two terms are the stated tolerance.  The third is
                   the error of computing y in fp32 before the one rounding to
                   the I/O dtype, which no fp32 implementation can avoid where
                   the numerator's terms cancel (|y| far below the terms,
                   e.g. in fp16's subnormal range, where 2 ulp is 2^-23):
                   y_abs = sum_i |term_i| / den, the output with every v and
                   the state's numerator replaced by their magnitudes (the
                   oracle on |v|, |num|), is the scale fp32 rounds against.
                   K_ARITH = 16 (2^-20 of y_abs) covers one call's arithmetic
                   (the worst element measured over the parity cases needs
                   11.8, at B=128, T=100, C=2048 fp16; 6.1 at the 14B width;
                   only a few hundred of 21 million need any); `calls` adds
                   2^-24 y_abs for each fp32 state
                   buffer the output's history passed through (each re-rounds
                   the carried state by up to half an fp32 ulp; 1024 decode
                   steps: up to 1023).
state:             num and den are brought to a shared max m* = max(p, p_ref)
                   (x_hat = x * e^{p - m*}); den must agree to
                   DEN_RTOL + calls * 2^-24 relative, and num/den (the running
                   average) to 2e-5 * max(max|v|, max|num_in/den_in|).  ``calls``
                   counts the fp32 state buffers the state passed through: each
                   store re-rounds (num, den, max) by up to half an fp32 ulp and
                   the error is carried into every later step (one forward call:
                   1; 1024 decode steps: 1024).
y_ref is the unrounded fp64 oracle output.
"""

import numpy as np
import torch

import oracle

Y_ABS_F32 = 2e-5
K_ARITH = 16
Y_REL_16 = 1e-3
AVG_ABS = 2e-5
DEN_RTOL = 1e-5

_MANT_BITS = {"f16": 10, "bf16": 7, "f32": 23}
_MIN_EXP = {"f16": -14, "bf16": -126, "f32": -126}


def ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of the fp16/bf16/fp32 grid at |x| (subnormal spacing below the normal range)."""
    m = _MANT_BITS[dtype]
    ax = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.where(ax > 0, np.floor(np.log2(np.where(ax > 0, ax, 1.0))), _MIN_EXP[dtype])
    e = np.maximum(e, _MIN_EXP[dtype])
    return np.ldexp(1.0, (e - m).astype(np.int64))


def to_f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def y_abs(k, v, w, u, state_in=None, nthreads: int = 1) -> np.ndarray:
    """sum_i |term_i| / den for every output of a forward call: the oracle's
    output with v and the state's numerator replaced by their magnitudes."""
    s = None
    if state_in is not None:
        s = to_f64(state_in).copy()
        s[0] = np.abs(s[0])
    y, _ = oracle.forward(k, np.abs(to_f64(v)), w, u, s, nthreads=nthreads)
    return y


def y_abs_gated(k, v, r, w, u, state_in=None, nthreads: int = 1) -> np.ndarray:
    """y_abs of the gated forward: sigmoid(r) times the ungated y_abs."""
    return oracle.sigmoid(r) * y_abs(k, v, w, u, state_in, nthreads)


def y_violations(y, y_ref, v, dtype: str, y_abs=None, calls: int = 0):
    """Boolean mask of elements outside the tolerance, and the bound used."""
    y, y_ref = to_f64(y), to_f64(y_ref)
    if dtype == "f32":
        bound = Y_ABS_F32 * float(np.max(np.abs(to_f64(v)))) if np.size(v) else 0.0
        bound = np.full_like(y_ref, bound)
    else:
        if y_abs is None:
            raise ValueError("the 16-bit gate needs y_abs (parity.y_abs)")
        bound = (2.0 * ulp(y_ref, dtype) + Y_REL_16 * np.abs(y_ref)
                 + (K_ARITH + calls) * 2.0 ** -24 * to_f64(y_abs))
    bad = ~(np.abs(y - y_ref) <= bound)  # NaN counts as a violation
    return bad, bound


def check_y(y, y_ref, v, dtype: str, what: str = "y", *, y_abs=None, calls: int = 0):
    bad, bound = y_violations(y, y_ref, v, dtype, y_abs, calls)
    if bad.any():
        y64, r64 = to_f64(y), to_f64(y_ref)
        idx = np.argwhere(bad)[:5]
        det = [(tuple(i), float(y64[tuple(i)]), float(r64[tuple(i)]), float(bound[tuple(i)]))
               for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"first (index, got, ref, bound): {det}")


def arith_excess(y, y_ref, y_abs, dtype: str) -> np.ndarray:
    """Per element, the error beyond the stated 16-bit tolerance in units of
    2^-24 y_abs (0 where the stated tolerance alone holds)."""
    y, y_ref = to_f64(y), to_f64(y_ref)
    ex = np.abs(y - y_ref) - (2.0 * ulp(y_ref, dtype) + Y_REL_16 * np.abs(y_ref))
    return np.where(ex > 0, ex / (2.0 ** -24 * to_f64(y_abs)), 0.0)


def state_errors(s, s_ref):
    """(relative den error, absolute error of num/den) per channel, after bringing
    both states to the shared max."""
    s, s_ref = to_f64(s), to_f64(s_ref)
    m = np.maximum(s[2], s_ref[2])
    e, e_ref = np.exp(s[2] - m), np.exp(s_ref[2] - m)
    a, b = s[0] * e, s[1] * e
    a_ref, b_ref = s_ref[0] * e_ref, s_ref[1] * e_ref
    den_rel = np.abs(b - b_ref) / b_ref
    avg = np.abs(a / b - a_ref / b_ref)
    return den_rel, avg


def check_state(s, s_ref, v, state_in=None, calls: int = 1, what: str = "state"):
    den_rtol = DEN_RTOL + calls * 2.0 ** -24
    den_rel, avg = state_errors(s, s_ref)
    scale = float(np.max(np.abs(to_f64(v)))) if np.size(v) else 0.0
    if state_in is not None:
        si = to_f64(state_in)
        with np.errstate(divide="ignore", invalid="ignore"):
            r = np.abs(si[0] / si[1])
        scale = max(scale, float(np.nanmax(np.where(np.isfinite(r), r, 0.0))))
    bad_den = ~(den_rel <= den_rtol)
    bad_avg = ~(avg <= AVG_ABS * scale)
    if bad_den.any() or bad_avg.any():
        raise AssertionError(
            f"{what}: den rel err max {np.nanmax(den_rel):.3e} (bound {den_rtol:.1e}, "
            f"{int(bad_den.sum())} bad); avg err max {np.nanmax(avg):.3e} "
            f"(bound {AVG_ABS * scale:.3e}, {int(bad_avg.sum())} bad)")
