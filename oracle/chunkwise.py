"""Chunkwise (WY / UT) restatement of Gated Delta Rule-2 and its reverse mode,
in numpy fp64.  TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages state that training is chunkwise, that normalising the state by the
cumulative decay folds the channel-wise decay into the two factors of each
rank-one erase, that the WY inverse is shared by the erase and write sides,
and that only the state crosses chunk borders ("Gated DeltaNet-2" LIT-802
review, "Key takeaways" 2, paper Secs. 3.3-3.4 and Apps. A-B; digg thread 9/).
They do not print the chunk equations; these are derived here from the
recurrence.  Per chunk of L tokens with entering state S (dk x dv), with the
cumulative log-decay G = cumsum(g) taken inclusively inside the chunk:

    Qb = q . e^G           (decay-scaled query)
    Kc = b . k . e^G       (erase factor)
    Kh = k . e^-G          (write factor)
    Kbar = k . e^(G_L - G) (state-update factor),   gam = e^(G_L)
    U  = w . v
    A  = strictly-lower(Kc Kh^T),   T = (I + A)^-1  (forward substitution)
    W  = T Kc,   U' = T U,   Delta = U' - W S
    P  = lower-incl(Qb Kh^T)
    O  = Qb S + P Delta
    S_next = diag(gam) S + Kbar^T Delta

Derivation: with S~_r = diag(e^-G_r) S_r, the recurrence becomes
S~_r = S~_{r-1} + Kh_r delta_r^T and delta_r = U_r - S~_{r-1}^T Kc_r, hence
(I + A) Delta = U - Kc S.  The read o_r = S_r^T q_r = S~_r^T Qb_r gives O.
The factors are used in the factored form; in fp64 this is exact as long as
|G| stays below ~700 inside a chunk, far beyond any decay the tests use.

The reverse mode is the chain rule applied to exactly these steps (in
reverse order); the gate-aware part is that b enters through Kc inside the
dot products that form A, so dA feeds dKc = ... + dA Kh with b inside, not a
scalar pulled outside.
"""

from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def _forward_substitution_inverse(A: np.ndarray) -> np.ndarray:
    """T = (I + A)^-1 for strictly-lower A, row by row:
    T_i = e_i - sum_{j<i} A_ij T_j."""
    L = A.shape[0]
    T = np.zeros_like(A)
    for i in range(L):
        T[i, i] = 1.0
        for j in range(i):
            T[i] -= A[i, j] * T[j]
    return T


def _chunk_factors(q, k, v, g, b, w):
    G = np.cumsum(g, axis=0)
    Ep, Em = np.exp(G), np.exp(-G)
    f = dict(G=G, Ep=Ep, Em=Em)
    f["Qb"] = q * Ep
    f["Kc"] = b * k * Ep
    f["Kh"] = k * Em
    f["Kbar"] = k * np.exp(G[-1][None, :] - G)
    f["gam"] = Ep[-1]
    f["U"] = w * v
    f["A"] = np.tril(f["Kc"] @ f["Kh"].T, -1)
    f["T"] = _forward_substitution_inverse(f["A"])
    f["W"] = f["T"] @ f["Kc"]
    f["Up"] = f["T"] @ f["U"]
    f["P"] = np.tril(f["Qb"] @ f["Kh"].T)
    return f


def forward(q, k, v, g, b, w, S0=None, *, chunk: int = 64, return_states: bool = False):
    """Chunkwise forward: (o, S_T) [and the list of chunk-entry states per (b, h)]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    states = {}
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[bi, h], dtype=np.float64)
            entry = []
            for c0 in range(0, T, chunk):
                c1 = min(T, c0 + chunk)
                sl = (bi, slice(c0, c1), h)
                f = _chunk_factors(q[sl], k[sl], v[sl], g[sl], b[sl], w[sl])
                entry.append(S.copy())
                D = f["Up"] - f["W"] @ S
                o[sl] = f["Qb"] @ S + f["P"] @ D
                S = f["gam"][:, None] * S + f["Kbar"].T @ D
            ST[bi, h] = S
            states[(bi, h)] = entry
    if return_states:
        return o, ST, states
    return o, ST


def backward(q, k, v, g, b, w, S0, dO, dST=None, *, chunk: int = 64) -> Dict[str, np.ndarray]:
    """Chunkwise reverse mode of L = <o, dO> + <S_T, dST>: dq, dk, dv, dg, db, dw, dS0."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _, _, states = forward(q, k, v, g, b, w, S0, chunk=chunk, return_states=True)
    out = {n: np.zeros(x.shape) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("db", b), ("dw", w))}
    out["dS0"] = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            dS = np.zeros((dk, dv)) if dST is None else np.array(dST[bi, h], dtype=np.float64)
            starts = list(range(0, T, chunk))
            for ci in reversed(range(len(starts))):
                c0 = starts[ci]
                c1 = min(T, c0 + chunk)
                sl = (bi, slice(c0, c1), h)
                S = states[(bi, h)][ci]
                f = _chunk_factors(q[sl], k[sl], v[sl], g[sl], b[sl], w[sl])
                Tm, W, Kc, Kh, Qb, Kbar, P = (f[n] for n in ("T", "W", "Kc", "Kh", "Qb", "Kbar", "P"))
                gam, U = f["gam"], f["U"]
                D = f["Up"] - W @ S
                dOc = dO[sl]
                # O = Qb S + P D ;  S_next = diag(gam) S + Kbar^T D
                dD = P.T @ dOc + Kbar @ dS
                dP = np.tril(dOc @ D.T)
                dQb = dOc @ S.T + dP @ Kh
                dKh = dP.T @ Qb
                dKbar = D @ dS.T
                dgam = (dS * S).sum(axis=1)
                dSc = Qb.T @ dOc + gam[:, None] * dS
                # D = U' - W S
                dUp = dD
                dW = -dD @ S.T
                dSc -= W.T @ dD
                # W = T Kc ; U' = T U
                dT = dW @ Kc.T + dUp @ U.T
                dKc = Tm.T @ dW
                dU = Tm.T @ dUp
                # T = (I + A)^-1 ;  A = strictly-lower(Kc Kh^T)
                dA = np.tril(-(Tm.T @ dT @ Tm.T), -1)
                dKc += dA @ Kh
                dKh += dA.T @ Kc
                # Kbar = Kh diag(gam)
                dKh += dKbar * gam[None, :]
                dgam += (dKbar * Kh).sum(axis=0)
                # elementwise factors
                Ep, Em = f["Ep"], f["Em"]
                qc, kc, bc, vc, wc = q[sl], k[sl], b[sl], v[sl], w[sl]
                dG = dQb * Qb + dKc * Kc - dKh * Kh
                dG[-1] += dgam * gam
                out["dq"][sl] = dQb * Ep
                out["db"][sl] = dKc * kc * Ep
                out["dk"][sl] = dKc * bc * Ep + dKh * Em
                out["dw"][sl] = dU * vc
                out["dv"][sl] = dU * wc
                # G = cumsum(g)  =>  dg = reverse cumsum of dG
                out["dg"][sl] = np.cumsum(dG[::-1], axis=0)[::-1]
                dS = dSc
            out["dS0"][bi, h] = dS
    return out
