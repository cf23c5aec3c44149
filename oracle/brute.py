"""TEST INFRASTRUCTURE ONLY: the WKV closed form evaluated term by term.

For tiny inputs this module evaluates, in 50-digit decimal arithmetic
(mpmath), the sums that define the RWKV-4 WKV output and state, with no
max-trick and no recurrence:

    y_t   = (e^{t w} A0 + sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u+k_t} v_t)
          / (e^{t w} D0 + sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u+k_t})
    A_out = e^{T w} A0 + sum_{i<T} e^{(T-1-i) w + k_i} v_i   (D_out with v = 1)

where (A0, D0) = (a e^p, b e^p) is the state given on entry (zero when none).
It pins the fp64 recurrence in ``wkv4_oracle.c``: the two share nothing but
the inputs.
"""

from __future__ import annotations

import mpmath
import numpy as np

mpmath.mp.dps = 50


def _mp(x) -> mpmath.mpf:
    return mpmath.mpf(float(x))


def closed_form(k, v, w, u, state_in=None):
    """k, v: [B, T, C]; w, u: [C]; state_in: [3, B, C] or None (fp64 arrays).

    Returns (y, A_out, D_out) as nested lists of mpmath numbers indexed
    [b][t][c] and [b][c]."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, C = k.shape
    y = [[[None] * C for _ in range(T)] for _ in range(B)]
    A_out = [[None] * C for _ in range(B)]
    D_out = [[None] * C for _ in range(B)]
    for b in range(B):
        for c in range(C):
            wc, uc = _mp(w[c]), _mp(u[c])
            if state_in is None:
                A0 = D0 = mpmath.mpf(0)
            else:
                e0 = mpmath.exp(_mp(state_in[2][b][c]))
                A0 = _mp(state_in[0][b][c]) * e0
                D0 = _mp(state_in[1][b][c]) * e0
            kk = [_mp(k[b, t, c]) for t in range(T)]
            vv = [_mp(v[b, t, c]) for t in range(T)]
            for t in range(T):
                num = mpmath.exp(t * wc) * A0
                den = mpmath.exp(t * wc) * D0
                for i in range(t):
                    e = mpmath.exp((t - 1 - i) * wc + kk[i])
                    num += e * vv[i]
                    den += e
                eb = mpmath.exp(uc + kk[t])
                y[b][t][c] = (num + eb * vv[t]) / (den + eb)
            num = mpmath.exp(T * wc) * A0
            den = mpmath.exp(T * wc) * D0
            for i in range(T):
                e = mpmath.exp((T - 1 - i) * wc + kk[i])
                num += e * vv[i]
                den += e
            A_out[b][c], D_out[b][c] = num, den
    return y, A_out, D_out
