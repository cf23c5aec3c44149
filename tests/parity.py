"""Parity gates between the CUDA path and the fp64 oracle.

y, fp32 I/O:       max |y - y_ref| <= 2e-5 * max|v|   (max over the call's v)
y, fp16/bf16 I/O:  |y - y_ref| <= 2 ulp_dtype(|y_ref|) + 1e-3 |y_ref| + 2e-5 * max|v|,
                   elementwise: the outputs are computed in fp32 and then rounded, so
                   the fp32 arithmetic's own allowance (the fp32 gate) is added to the
                   rounding allowance; without it outputs near zero, where the fp32
                   numerator cancels (|y| < 1e-4, in fp16's subnormal range), miss by
                   an ulp or two of fp16
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

Y_ABS_F32 = 2e-5
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


def y_violations(y, y_ref, v, dtype: str):
    """Boolean mask of elements outside the tolerance, and the bound used."""
    y, y_ref = to_f64(y), to_f64(y_ref)
    if dtype == "f32":
        bound = Y_ABS_F32 * float(np.max(np.abs(to_f64(v)))) if np.size(v) else 0.0
        bound = np.full_like(y_ref, bound)
    else:
        vmax = float(np.max(np.abs(to_f64(v)))) if np.size(v) else 0.0
        bound = 2.0 * ulp(y_ref, dtype) + Y_REL_16 * np.abs(y_ref) + Y_ABS_F32 * vmax
    bad = ~(np.abs(y - y_ref) <= bound)  # NaN counts as a violation
    return bad, bound


def check_y(y, y_ref, v, dtype: str, what: str = "y"):
    bad, bound = y_violations(y, y_ref, v, dtype)
    if bad.any():
        y64, r64 = to_f64(y), to_f64(y_ref)
        idx = np.argwhere(bad)[:5]
        det = [(tuple(i), float(y64[tuple(i)]), float(r64[tuple(i)]), float(bound[tuple(i)]))
               for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"first (index, got, ref, bound): {det}")


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
