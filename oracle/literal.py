"""The Gated Delta Rule-2 update in the matrix form the pages print, evaluated in
exact rational arithmetic.  TEST INFRASTRUCTURE ONLY.

"Gated DeltaNet-2" LIT-802 review, "Key takeaways" 1 (paper Sec. 3.1,
Eqs. 8-10); wispaper.ai blog, "Methodology: Gated Delta Rule-2":

    S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T

Here the erase operator E_t = I - k_t (b_t . k_t)^T is built as a dk x dk
matrix and multiplied out, exactly as printed, unlike the oracle's token loop
(which reads, subtracts and writes a rank-one correction).  D_t's diagonal is
given directly as rationals alpha_t = exp(g_t).  The read is o_t = S_t^T q_t.
"""

from __future__ import annotations

from fractions import Fraction
from typing import List, Sequence, Tuple

Mat = List[List[Fraction]]


def _matmul(X: Mat, Y: Mat) -> Mat:
    n, m, p = len(X), len(Y), len(Y[0])
    return [[sum((X[i][l] * Y[l][j] for l in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def step(S: Mat, q: Sequence[Fraction], k: Sequence[Fraction], v: Sequence[Fraction],
         alpha: Sequence[Fraction], b: Sequence[Fraction], w: Sequence[Fraction]
         ) -> Tuple[Mat, List[Fraction]]:
    dk, dv = len(k), len(v)
    E = [[(Fraction(1) if i == j else Fraction(0)) - k[i] * (b[j] * k[j]) for j in range(dk)]
         for i in range(dk)]
    DS = [[alpha[i] * S[i][j] for j in range(dv)] for i in range(dk)]
    ES = _matmul(E, DS)
    Snew = [[ES[i][j] + k[i] * (w[j] * v[j]) for j in range(dv)] for i in range(dk)]
    o = [sum((Snew[i][j] * q[i] for i in range(dk)), Fraction(0)) for j in range(dv)]
    return Snew, o


def run(S0: Mat, seq) -> Tuple[Mat, List[List[Fraction]]]:
    """seq: list of dicts with keys q, k, v, alpha, b, w (lists of Fractions)."""
    S = [row[:] for row in S0]
    outs = []
    for tok in seq:
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["b"], tok["w"])
        outs.append(o)
    return S, outs
