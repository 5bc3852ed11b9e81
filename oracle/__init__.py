"""fp64 CPU oracle for the Gated Delta Rule-2 operator.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls, links or loads anything here, and nothing here imports the CUDA
library: the two share no code.

Contents (sources: "Gated DeltaNet-2: Decoupling Erase and Write in Linear
Attention", anthology-of-the-sota LIT-802 review, "Key takeaways" 1-2, paper
Sec. 3.1 Eqs. 8-10, Secs. 3.3-3.4, App. A.5, App. D.6; digg thread 7/-11/):

* ``forward`` / ``backward`` - the token-by-token recurrence and its reverse
  mode (C, fp64, threads over (b, h)): the plain definition.
* ``kda_forward`` / ``gdn_forward`` - KDA and Gated DeltaNet written in their
  own matrix form, for the tie identities.
* ``chunkwise`` - the chunkwise (WY/UT) restatement and its reverse mode, in
  numpy fp64, pinned against the token loop.
* ``fd`` - central finite differences of the token loop.
* ``literal`` - the printed matrix form of the update evaluated in exact
  rational arithmetic, for tiny golden cases.

Every function takes and returns float64 numpy arrays in the operator's
layouts: [B, T, H, D] activations and gates, [B, H, dk, dv] states.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.gdn2_oracle_forward.argtypes = [dp] * 9 + [i] * 6
        lib.gdn2_oracle_backward.argtypes = [dp] * 16 + [i] * 7
        lib.kda_oracle_forward.argtypes = [dp] * 8 + [i] * 6
        lib.gdn_oracle_forward.argtypes = [dp] * 8 + [i] * 6
        for f in (lib.gdn2_oracle_forward, lib.gdn2_oracle_backward,
                  lib.kda_oracle_forward, lib.gdn_oracle_forward):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _c(x: Optional[np.ndarray]):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x: Optional[np.ndarray]):
    if x is None:
        return ctypes.POINTER(ctypes.c_double)()
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(q, k, v, g, b, w, S0=None, *, nthreads: Optional[int] = None
            ) -> Tuple[np.ndarray, np.ndarray]:
    """Token-wise forward: returns (o [B,T,H,dv], S_T [B,H,dk,dv])."""
    q, k, v, g, b, w, S0 = map(_c, (q, k, v, g, b, w, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = _load().gdn2_oracle_forward(_p(q), _p(k), _p(v), _p(g), _p(b), _p(w), _p(S0),
                                     _p(o), _p(ST), B, T, H, dk, dv,
                                     nthreads or default_threads())
    if rc:
        raise ValueError("gdn2_oracle_forward: bad dimensions")
    return o, ST


def backward(q, k, v, g, b, w, S0, dO, dST=None, *, ckpt: int = 64,
             nthreads: Optional[int] = None):
    """Token-wise reverse mode of L = <o, dO> + <S_T, dST>.

    Returns dict dq, dk, dv, dg, db, dw, dS0."""
    q, k, v, g, b, w, S0, dO, dST = map(_c, (q, k, v, g, b, w, S0, dO, dST))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {n: np.zeros(x.shape) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("db", b), ("dw", w))}
    out["dS0"] = np.zeros((B, H, dk, dv))
    rc = _load().gdn2_oracle_backward(
        _p(q), _p(k), _p(v), _p(g), _p(b), _p(w), _p(S0), _p(dO), _p(dST),
        _p(out["dq"]), _p(out["dk"]), _p(out["dv"]), _p(out["dg"]), _p(out["db"]),
        _p(out["dw"]), _p(out["dS0"]), B, T, H, dk, dv, ckpt, nthreads or default_threads())
    if rc:
        raise ValueError("gdn2_oracle_backward: bad arguments")
    return out


def kda_forward(q, k, v, g, beta, S0=None, *, nthreads: Optional[int] = None):
    """KDA: S_t = (I - beta k k^T) Diag(exp g) S_{t-1} + beta k v^T; o = S_t^T q."""
    q, k, v, g, beta, S0 = map(_c, (q, k, v, g, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = _load().kda_oracle_forward(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(S0), _p(o),
                                    _p(ST), B, T, H, dk, dv, nthreads or default_threads())
    if rc:
        raise ValueError("kda_oracle_forward: bad dimensions")
    return o, ST


def gdn_forward(q, k, v, alpha_log, beta, S0=None, *, nthreads: Optional[int] = None):
    """Gated DeltaNet: S_t = exp(a_t)(I - beta k k^T) S_{t-1} + beta k v^T; o = S_t^T q."""
    q, k, v, alpha_log, beta, S0 = map(_c, (q, k, v, alpha_log, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = _load().gdn_oracle_forward(_p(q), _p(k), _p(v), _p(alpha_log), _p(beta), _p(S0),
                                    _p(o), _p(ST), B, T, H, dk, dv,
                                    nthreads or default_threads())
    if rc:
        raise ValueError("gdn_oracle_forward: bad dimensions")
    return o, ST
