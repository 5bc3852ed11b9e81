"""Central finite differences of a forward function.  TEST INFRASTRUCTURE ONLY.

The pages check their chunkwise gradients against a token-wise reference in
fp64 ("Gated DeltaNet-2" LIT-802 review, "Key takeaways" 2, paper App. D.6).
This module gives the calculus-level check under that: dL/dx for
L = <o, dO> + <S_T, dST>, one input element at a time, with step h.
"""

from __future__ import annotations

from typing import Callable, Dict, Optional, Sequence

import numpy as np

from . import forward as _gdr2_forward

GDR2_NAMES = ("q", "k", "v", "g", "b", "w", "S0")


def _loss(fn, args, dO, dST) -> float:
    o, ST = fn(*args)
    val = float(np.sum(o * dO))
    if dST is not None:
        val += float(np.sum(ST * dST))
    return val


def gradients(inputs: Dict[str, np.ndarray], dO: np.ndarray, dST: Optional[np.ndarray] = None,
              h: float = 1e-6, *, fn: Optional[Callable] = None,
              names: Sequence[str] = GDR2_NAMES) -> Dict[str, np.ndarray]:
    """(L(x+h) - L(x-h)) / 2h for every element of every named input.

    ``fn(*[inputs[n] for n in names]) -> (o, S_T)``; default: the token-wise
    Gated Delta Rule-2 forward over (q, k, v, g, b, w, S0)."""
    if fn is None:
        fn = lambda *a: _gdr2_forward(*a, nthreads=1)  # noqa: E731
    base = [np.array(inputs[n], dtype=np.float64, copy=True) for n in names]
    grads = {}
    for idx, n in enumerate(names):
        x = base[idx]
        gr = np.zeros_like(x)
        flat, gflat = x.reshape(-1), gr.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = _loss(fn, base, dO, dST)
            flat[i] = keep - h
            lm = _loss(fn, base, dO, dST)
            flat[i] = keep
            gflat[i] = (lp - lm) / (2 * h)
        grads["d" + n] = gr
    return grads
