"""Writes closed_form_tiny.json: WKV-4 outputs of a tiny input, evaluated as
the literal closed-form sums in 50-digit arithmetic by ``oracle.brute``.

Citation: the output and state are the decayed, bonus-weighted averages of v
with weights e^k that define the RWKV-4 WKV time mix; the state on entry is
the (num, den, max) triple of "RWKV in a self-built engine: a second
non-attention paradigm (WKV/RNN)", Methods table, "Precision" row.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
from oracle import brute  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_form_tiny.json")


def main():
    # hand-picked values: exact in binary, one spike, one huge and one tiny decay
    k = np.array([[[0.5, -1.25, 2.0], [30.0, 0.75, -3.5], [-2.0, 1.5, 0.25],
                   [1.0, -0.5, 30.0], [0.0, 2.25, -1.0]]])
    v = np.array([[[1.0, -0.5, 0.25], [-2.0, 1.5, 0.75], [0.5, 0.125, -1.25],
                   [1.75, -1.0, 2.0], [-0.25, 0.875, 0.5]]])
    w = np.array([-0.0625, -7.375, -0.00048828125])
    u = np.array([0.5, -3.0, 2.5])
    state = np.array([[[0.75, -1.5, 0.3125]], [[1.25, 0.625, 1.875]], [[-0.5, 1.0, -2.0]]])
    cases = []
    for s in (None, state):
        y, A, D = brute.closed_form(k, v, w, u, s)
        cases.append({
            "state_in": None if s is None else s.tolist(),
            "y": [[[str(x) for x in row] for row in yb] for yb in y],
            "A_out": [[str(x) for x in row] for row in A],
            "D_out": [[str(x) for x in row] for row in D],
        })
    doc = {
        "what": "RWKV-4 WKV forward, B=1 T=5 C=3, closed-form sums at 50 digits",
        "cite": "RWKV in a self-built engine: a second non-attention paradigm (WKV/RNN), "
                "Methods table 'Precision' row (num/den/max state); closed form of the "
                "RWKV-4 WKV time mix",
        "generator": "tests/golden/make_golden.py (calls oracle.brute only)",
        "k": k.tolist(), "v": v.tolist(), "w": w.tolist(), "u": u.tolist(),
        "cases": cases,
    }
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
