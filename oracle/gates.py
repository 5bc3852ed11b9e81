"""The fused gate prologue, for the oracle.  TEST INFRASTRUCTURE ONLY (see the
package docstring).

"Gated DeltaNet-2" (LIT-802 review, "Key takeaways" 1) makes the erase gate b
and the write gate w sigmoid outputs and the decay a log-sigmoid; its Table 5
also runs the erase gate as 2 sigmoid, for erase eigenvalues in [-1, 1].  Here
the operator takes the pre-activation logits x_g, x_b, x_w:

    g = log sigmoid(x_g),   b = s sigmoid(x_b) (s = 1 or 2),   w = sigmoid(x_w)

in fp64, and the gradients of the logits follow by the chain rule from the
token loop's (``oracle.backward``):

    dx_g = dg sigmoid(-x_g),   dx_b = db s sigma_b (1 - sigma_b),   dx_w = dw sigma_w (1 - sigma_w).
"""

from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np

from . import backward as _backward
from . import forward as _forward


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def activate(xg, xb, xw, b_scale: float = 1.0) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(g, b, w) from the logits; log sigmoid written as -log(1 + e^-x) in a
    form that does not overflow."""
    g = np.minimum(xg, 0.0) - np.log1p(np.exp(-np.abs(xg)))
    return g, b_scale * _sigmoid(xb), _sigmoid(xw)


def forward(q, k, v, xg, xb, xw, S0: Optional[np.ndarray] = None, *, b_scale: float = 1.0):
    g, b, w = activate(xg, xb, xw, b_scale)
    return _forward(q, k, v, g, b, w, S0)


def backward(q, k, v, xg, xb, xw, S0, dO, dST=None, *, b_scale: float = 1.0,
             ckpt: int = 64) -> Dict[str, np.ndarray]:
    g, b, w = activate(xg, xb, xw, b_scale)
    r = _backward(q, k, v, g, b, w, S0, dO, dST, ckpt=ckpt)
    sb, sw = _sigmoid(xb), _sigmoid(xw)
    r["dg"] = r["dg"] * _sigmoid(-xg)
    r["db"] = r["db"] * b_scale * sb * (1.0 - sb)
    r["dw"] = r["dw"] * sw * (1.0 - sw)
    return r
