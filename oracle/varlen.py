"""Packed variable-length sequences, for the oracle.  TEST INFRASTRUCTURE ONLY
(see the package docstring).

N sequences lie back to back along the token axis of one batch row, sequence
n at tokens cu_seqlens[n] .. cu_seqlens[n + 1] - 1, each with its own initial
state S0[n] and final state S_T[n].  The recurrence ("Gated DeltaNet-2",
LIT-802 review, "Key takeaways" 1) runs over each sequence on its own: no
state crosses from one sequence to the next.  So the packed forward and
backward are the token loop (``oracle.forward`` / ``oracle.backward``) applied
to each slice, with the results put back in place; an empty sequence has
S_T = S0 and dS0 = dS_T.

Layouts: q, k, g, b [1, T, H, d_k]; v, w, dO [1, T, H, d_v]; S0, dST
[N, H, d_k, d_v].
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from . import backward as _backward
from . import forward as _forward


def _slices(cu: Sequence[int]):
    cu = [int(x) for x in cu]
    if cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must rise from 0")
    return list(zip(cu[:-1], cu[1:]))


def forward(q, k, v, g, b, w, cu_seqlens, S0: Optional[np.ndarray] = None):
    """(o [1, T, H, d_v], S_T [N, H, d_k, d_v])."""
    sl = _slices(cu_seqlens)
    N, H, dk, dv = len(sl), q.shape[2], q.shape[3], v.shape[3]
    o = np.zeros(v.shape[:3] + (dv,))
    ST = np.zeros((N, H, dk, dv))
    for n, (a, e) in enumerate(sl):
        s0 = None if S0 is None else S0[n:n + 1]
        if e == a:
            ST[n] = 0.0 if S0 is None else S0[n]
            continue
        o_n, ST_n = _forward(*(x[:, a:e] for x in (q, k, v, g, b, w)), s0)
        o[:, a:e] = o_n
        ST[n] = ST_n[0]
    return o, ST


def backward(q, k, v, g, b, w, cu_seqlens, S0, dO, dST=None, *, ckpt: int = 64) -> Dict[str, np.ndarray]:
    """Gradients dq, dk, dv, dg, db, dw (packed layouts) and dS0 [N, H, d_k, d_v]."""
    sl = _slices(cu_seqlens)
    N, H, dk, dv = len(sl), q.shape[2], q.shape[3], v.shape[3]
    out = {n: np.zeros(x.shape) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("db", b),
                                                ("dw", w))}
    out["dS0"] = np.zeros((N, H, dk, dv))
    for n, (a, e) in enumerate(sl):
        if e == a:
            out["dS0"][n] = 0.0 if dST is None else dST[n]
            continue
        s0 = None if S0 is None else S0[n:n + 1]
        dst = None if dST is None else dST[n:n + 1]
        r = _backward(*(x[:, a:e] for x in (q, k, v, g, b, w)), s0, dO[:, a:e], dst, ckpt=ckpt)
        for name in ("dq", "dk", "dv", "dg", "db", "dw"):
            out[name][:, a:e] = r[name]
        out["dS0"][n] = r["dS0"][0]
    return out
