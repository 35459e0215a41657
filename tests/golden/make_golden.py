"""Writes the hand-derivable worked examples in this folder.

The pages print no worked example, so these fixtures come from cases whose
result follows from the definitions alone, evaluated in exact rational
arithmetic (Python ``fractions``).  This script calls neither the oracle nor
the CUDA library.

Why the cases are exact: a matrix with one non-zero singular value (a single
row or column) normalised by its Frobenius norm has that singular value equal
to 1, and a diagonal matrix keeps every iterate diagonal.  Newton-Schulz then
reduces to the scalar quintic p(s) = a s + b s^3 + c s^5 applied ``steps``
times to each singular value / diagonal entry.  With eps = 0 every quantity up
to the sqrt(max(rows, cols)) factor of the update scale is rational.

Run:  python tests/golden/make_golden.py
"""
from __future__ import annotations

import json
import math
from fractions import Fraction as F
from pathlib import Path

A, B, C = F("3.4445"), F("-4.7750"), F("2.0315")


def p(s: F) -> F:
    return A * s + B * s ** 3 + C * s ** 5


def f(s: F, steps: int) -> F:
    for _ in range(steps):
        s = p(s)
    return s


def as_str(x) -> str:
    return repr(float(x)) if not isinstance(x, str) else x


def case_rank1(rows, cols, g, b, w, mu, lr, wd, steps):
    """G, B, W given as flat lists for a 1 x n or n x 1 matrix."""
    g = [F(x) for x in g]
    b = [F(x) for x in b]
    mu = F(mu)
    b_new = [mu * bi + gi for bi, gi in zip(b, g)]
    u = [gi + mu * bi for gi, bi in zip(g, b_new)]
    norm2 = sum(x * x for x in u)
    # the cases are chosen so that the norm is rational
    norm = F(math.isqrt(norm2.numerator), math.isqrt(norm2.denominator))
    assert norm * norm == norm2
    x0 = [x / norm for x in u]
    fk = f(F(1), steps)
    o = [fk * x for x in x0]
    scale = 0.2 * math.sqrt(max(rows, cols))
    decay = 1 - F(lr) * F(wd)
    w_new = [float(decay * F(wi)) - float(F(lr) * fk * xi) * scale for wi, xi in zip(w, x0)]
    return {
        "rows": rows, "cols": cols, "mu": float(mu), "lr": lr, "wd": wd, "eps": 0.0,
        "ns_steps": steps, "nesterov": True,
        "G": [float(x) for x in g], "B": [float(x) for x in b], "W": w,
        "B_new": [float(x) for x in b_new], "U": [float(x) for x in u],
        "O": [float(x) for x in o], "W_new": w_new,
        "f_steps_at_1": float(fk),
    }


def case_diag(d, steps, lr, wd, w):
    """G = diag(d), B = 0, mu = 0: U = G, the NS acts entrywise on d/||d||."""
    d = [F(x) for x in d]
    norm2 = sum(x * x for x in d)
    norm = F(math.isqrt(norm2.numerator), math.isqrt(norm2.denominator))
    assert norm * norm == norm2
    n = len(d)
    o = [f(x / norm, steps) if x >= 0 else -f(-x / norm, steps) for x in d]
    scale = 0.2 * math.sqrt(n)
    decay = 1 - F(lr) * F(wd)
    Wn = []
    for i in range(n):
        row = []
        for j in range(n):
            oij = o[i] if i == j else F(0)
            row.append(float(decay * F(w[i][j])) - float(F(lr) * oij) * scale)
        Wn.append(row)
    return {
        "rows": n, "cols": n, "mu": 0.0, "lr": lr, "wd": wd, "eps": 0.0,
        "ns_steps": steps, "nesterov": True,
        "G": [[float(d[i]) if i == j else 0.0 for j in range(n)] for i in range(n)],
        "B": [[0.0] * n for _ in range(n)], "W": w,
        "O_diag": [float(x) for x in o], "W_new": Wn,
    }


def main():
    here = Path(__file__).parent
    cases = {
        "rank1_row_1x2": case_rank1(1, 2, ["3", "4"], ["0", "0"], [0.5, -0.25],
                                    "0.95", 0.02, 0.1, 5),
        "rank1_col_2x1": case_rank1(2, 1, ["3", "4"], ["0", "0"], [0.5, -0.25],
                                    "0.95", 0.02, 0.1, 5),
        # non-zero momentum: B' = 0.5*(2,-1)... chosen so that U = (6, 8)
        "rank1_row_momentum_1x2": case_rank1(1, 2, ["4", "6"], ["0", "-4"], [0.1, 0.2],
                                             "0.5", 0.02, 0.1, 3),
        "diag_2x2": case_diag(["3", "-4"], 5, 0.02, 0.1, [[0.25, 0.5], [-0.5, 0.125]]),
        "diag_3x3": case_diag(["2", "3", "6"], 5, 0.01, 0.2,
                              [[0.1, 0.0, 0.2], [0.0, -0.3, 0.0], [0.4, 0.0, 0.5]]),
    }
    doc = {
        "source": "derived from the definitions (no worked example is printed on the pages); "
                  "see make_golden.py for the derivation",
        "coefficients": [str(A), str(B), str(C)],
        "cases": cases,
    }
    (here / "worked_examples.json").write_text(json.dumps(doc, indent=1) + "\n")


if __name__ == "__main__":
    main()
