"""Grouped value heads, for the oracle.  TEST INFRASTRUCTURE ONLY (see the
package docstring).

H_v value heads over H query/key heads ("Gated DeltaNet-2", LIT-802 review,
"Where the hedges are": the write gate has H_v d_v outputs, the erase gate
H d_k).  Value head j reads query/key head j / G (G = H_v / H consecutive value
heads per key head): q, k, g, b are [B, T, H, d_k]; v, w, dO are
[B, T, H_v, d_v]; states are [B, H_v, d_k, d_v].  Each value head is the plain
recurrence with its key head's q, k, g, b, so the grouped forward is the token
loop (``oracle.forward``) on q, k, g, b repeated G times along the head axis,
and the gradients of q, k, g, b are the sums over each key head's G copies.
"""

from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from . import backward as _backward
from . import forward as _forward

_KEY_SIDE = ("q", "k", "g", "b")


def _repeat(x: np.ndarray, G: int) -> np.ndarray:
    return np.repeat(x, G, axis=2)


def forward(q, k, v, g, b, w, S0: Optional[np.ndarray] = None):
    """(o [B, T, H_v, d_v], S_T [B, H_v, d_k, d_v])."""
    G = v.shape[2] // q.shape[2]
    return _forward(_repeat(q, G), _repeat(k, G), v, _repeat(g, G), _repeat(b, G), w, S0)


def backward(q, k, v, g, b, w, S0, dO, dST=None, *, ckpt: int = 64) -> Dict[str, np.ndarray]:
    """Gradients dq, dk, dg, db [B, T, H, d_k], dv, dw [B, T, H_v, d_v], dS0."""
    B, T, H, dk = q.shape
    G = v.shape[2] // H
    r = _backward(_repeat(q, G), _repeat(k, G), v, _repeat(g, G), _repeat(b, G), w, S0, dO, dST,
                  ckpt=ckpt)
    for n in _KEY_SIDE:
        r["d" + n] = r["d" + n].reshape(B, T, H, G, dk).sum(axis=3)
    return r
