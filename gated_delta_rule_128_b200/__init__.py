"""Python binding of libgdn2.so, the B200 (sm_100a) Gated Delta Rule-2 operator.

Argument marshalling only: every step of the operator runs in the CUDA
library.  There is no CPU path; importing works anywhere, but the first call
raises if ``libgdn2.so`` has not been built (``python -m
gated_delta_rule_128_b200.build``).

Two layers:

* ``gdn2_fwd``, ``gdn2_bwd``, ``gdn2_decode_step`` (and their ``_ex`` forms with
  the gates' own type), ``gdn2_workspace_bytes``,
  ``gdn2_get_device_status``: the C entry points of ``include/gdn2.h`` under
  the same names, taking torch tensors (or None) where the C call takes
  pointers, and raising ``Gdn2Error`` on a non-zero status.
* ``forward``, ``backward``, ``decode_step``: allocate outputs and workspace
  with torch (device memory is PyTorch's job here) and call the above on the
  current CUDA stream; ``forward`` and ``backward`` then read the device
  status word and raise on a recorded error unless called with check=False.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdn2.so")

GDN2_IO_F32 = 0
GDN2_IO_BF16 = 1
GDN2_GATE_LOGITS = 0x100   # g, b, w are logits: g = logsigmoid, b = sigmoid (x2 with B_X2), w = sigmoid
GDN2_GATE_B_X2 = 0x200
GATE_FLAGS = {"activated": 0, "logits": GDN2_GATE_LOGITS, "logits_b2": GDN2_GATE_LOGITS | GDN2_GATE_B_X2}
STATUS = {0: "GDN2_OK", 1: "GDN2_ERR_INVALID_ARG", 2: "GDN2_ERR_UNSUPPORTED",
          3: "GDN2_ERR_WORKSPACE", 4: "GDN2_ERR_CUDA", 5: "GDN2_ERR_TIMEOUT",
          6: "GDN2_ERR_RANGE"}


class Gdn2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().gdn2_status_string(status).decode()
        super().__init__(f"{fn} returned {STATUS.get(status, status)}: {msg}")


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libgdn2.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run "
                               "`python -m gated_delta_rule_128_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.gdn2_workspace_bytes.argtypes = [i] * 8
        L.gdn2_workspace_bytes.restype = sz
        L.gdn2_fwd.argtypes = [vp] * 10 + [sz] + [i] * 7 + [vp]
        L.gdn2_fwd.restype = i
        L.gdn2_bwd.argtypes = [vp] * 17 + [sz, i] + [i] * 7 + [vp]
        L.gdn2_bwd.restype = i
        L.gdn2_decode_step.argtypes = [vp] * 8 + [i] * 5 + [vp]
        L.gdn2_workspace_bytes_ex.argtypes = [i] * 10
        L.gdn2_workspace_bytes_ex.restype = sz
        L.gdn2_fwd_ex.argtypes = [vp] * 10 + [sz] + [i] * 9 + [vp]
        L.gdn2_fwd_ex.restype = i
        L.gdn2_bwd_ex.argtypes = [vp] * 17 + [sz, i] + [i] * 9 + [vp]
        L.gdn2_bwd_ex.restype = i
        L.gdn2_decode_step_ex.argtypes = [vp] * 8 + [i] * 7 + [vp]
        L.gdn2_decode_step_ex.restype = i
        L.gdn2_workspace_bytes_varlen.argtypes = [i] * 10
        L.gdn2_workspace_bytes_varlen.restype = sz
        L.gdn2_fwd_varlen.argtypes = [vp] * 10 + [sz, vp] + [i] * 9 + [vp]
        L.gdn2_fwd_varlen.restype = i
        L.gdn2_bwd_varlen.argtypes = [vp] * 17 + [sz, i, vp] + [i] * 9 + [vp]
        L.gdn2_bwd_varlen.restype = i
        L.gdn2_decode_step.restype = i
        L.gdn2_get_device_status.argtypes = [vp]
        L.gdn2_get_device_status.restype = i
        L.gdn2_selftest_timeout.argtypes = [ctypes.c_longlong, vp]
        L.gdn2_selftest_timeout.restype = i
        L.gdn2_status_string.argtypes = [i]
        L.gdn2_status_string.restype = ctypes.c_char_p
        L.gdn2_version.argtypes = []
        L.gdn2_version.restype = i
        L.gdn2_fwd_noalloc.argtypes = [vp] * 9 + [i] * 7 + [vp]
        L.gdn2_fwd_noalloc.restype = i
        L.gdn2_kernel_launches.argtypes = []
        L.gdn2_kernel_launches.restype = ctypes.c_ulonglong
        L.gdn2_set_kernel_timer.argtypes = [i]
        L.gdn2_set_kernel_timer.restype = None
        L.gdn2_kernel_kinds.argtypes = []
        L.gdn2_kernel_kinds.restype = i
        L.gdn2_kernel_name.argtypes = [i]
        L.gdn2_kernel_name.restype = ctypes.c_char_p
        L.gdn2_kernel_times.argtypes = [vp, vp, i]
        L.gdn2_kernel_times.restype = i
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libgdn2 must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _io_of(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN2_IO_BF16
    if t.dtype == torch.float32:
        return GDN2_IO_F32
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _gate_io_of(g: torch.Tensor, b: torch.Tensor, w: torch.Tensor, gates: str = "activated") -> int:
    """The gate_io argument: the gates' dtype, or-ed with the flags of the
    gate encoding ("activated" values, "logits", or "logits_b2")."""
    if not (g.dtype == b.dtype == w.dtype):
        raise TypeError(f"g, b, w must share one dtype, got {g.dtype}, {b.dtype}, {w.dtype}")
    if gates not in GATE_FLAGS:
        raise ValueError(f"gates must be one of {sorted(GATE_FLAGS)}, got {gates!r}")
    if g.dtype == torch.bfloat16:
        return GDN2_IO_BF16 | GATE_FLAGS[gates]
    if g.dtype == torch.float32:
        return GDN2_IO_F32 | GATE_FLAGS[gates]
    raise TypeError(f"g/b/w must be float32 or bfloat16, got {g.dtype}")


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, rc: int):
    if rc != 0:
        raise Gdn2Error(fn, rc)


# ------------------------------------------------------------- C entry points

def gdn2_workspace_bytes(B, T, H, d_k, d_v, chunk, io, for_bwd) -> int:
    return int(lib().gdn2_workspace_bytes(B, T, H, d_k, d_v, chunk, io, int(for_bwd)))


def gdn2_fwd(q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, B, T, H, d_k, d_v, chunk, io,
             stream=None):
    rc = lib().gdn2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                        _ptr(ST), _ptr(ws), ws_bytes, B, T, H, d_k, d_v, chunk, io,
                        _stream(stream))
    _check("gdn2_fwd", rc)


def gdn2_fwd_noalloc(q, k, v, g, b, w, S0, o, ST, B, T, H, d_k, d_v, chunk, io, stream=None):
    rc = lib().gdn2_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0),
                                _ptr(o), _ptr(ST), B, T, H, d_k, d_v, chunk, io, _stream(stream))
    _check("gdn2_fwd_noalloc", rc)


def gdn2_bwd(q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes,
             ws_has_fwd, B, T, H, d_k, d_v, chunk, io, stream=None):
    rc = lib().gdn2_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO),
                        _ptr(dST), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(db), _ptr(dw),
                        _ptr(dS0), _ptr(ws), ws_bytes, int(ws_has_fwd), B, T, H, d_k, d_v, chunk,
                        io, _stream(stream))
    _check("gdn2_bwd", rc)


def gdn2_workspace_bytes_ex(B, T, H, H_v, d_k, d_v, chunk, io, gate_io, for_bwd) -> int:
    return int(lib().gdn2_workspace_bytes_ex(B, T, H, H_v, d_k, d_v, chunk, io, gate_io, int(for_bwd)))


def gdn2_fwd_ex(q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, B, T, H, H_v, d_k, d_v, chunk, io,
                gate_io, stream=None):
    rc = lib().gdn2_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                           _ptr(ST), _ptr(ws), ws_bytes, B, T, H, H_v, d_k, d_v, chunk, io, gate_io,
                           _stream(stream))
    _check("gdn2_fwd_ex", rc)


def gdn2_bwd_ex(q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes,
                ws_has_fwd, B, T, H, H_v, d_k, d_v, chunk, io, gate_io, stream=None):
    rc = lib().gdn2_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO),
                           _ptr(dST), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(db), _ptr(dw),
                           _ptr(dS0), _ptr(ws), ws_bytes, int(ws_has_fwd), B, T, H, H_v, d_k, d_v,
                           chunk, io, gate_io, _stream(stream))
    _check("gdn2_bwd_ex", rc)


def gdn2_decode_step_ex(q, k, v, g, b, w, S, o, N, H, H_v, d_k, d_v, io, gate_io, stream=None):
    rc = lib().gdn2_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S),
                                   _ptr(o), N, H, H_v, d_k, d_v, io, gate_io, _stream(stream))
    _check("gdn2_decode_step_ex", rc)


def gdn2_workspace_bytes_varlen(N, T, H, H_v, d_k, d_v, chunk, io, gate_io, for_bwd) -> int:
    return int(lib().gdn2_workspace_bytes_varlen(N, T, H, H_v, d_k, d_v, chunk, io, gate_io,
                                                 int(for_bwd)))


def gdn2_fwd_varlen(q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, cu_seqlens, N, T, H, H_v, d_k, d_v,
                    chunk, io, gate_io, stream=None):
    rc = lib().gdn2_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0),
                               _ptr(o), _ptr(ST), _ptr(ws), ws_bytes, _ptr(cu_seqlens), N, T, H,
                               H_v, d_k, d_v, chunk, io, gate_io, _stream(stream))
    _check("gdn2_fwd_varlen", rc)


def gdn2_bwd_varlen(q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes,
                    ws_has_fwd, cu_seqlens, N, T, H, H_v, d_k, d_v, chunk, io, gate_io,
                    stream=None):
    rc = lib().gdn2_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0),
                               _ptr(dO), _ptr(dST), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                               _ptr(db), _ptr(dw), _ptr(dS0), _ptr(ws), ws_bytes, int(ws_has_fwd),
                               _ptr(cu_seqlens), N, T, H, H_v, d_k, d_v, chunk, io, gate_io,
                               _stream(stream))
    _check("gdn2_bwd_varlen", rc)


def gdn2_decode_step(q, k, v, g, b, w, S, o, N, H, d_k, d_v, io, stream=None):
    rc = lib().gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S),
                                _ptr(o), N, H, d_k, d_v, io, _stream(stream))
    _check("gdn2_decode_step", rc)


def gdn2_get_device_status(stream=None) -> int:
    return int(lib().gdn2_get_device_status(_stream(stream)))


def gdn2_selftest_timeout(limit_cycles: int = 2_000_000, stream=None) -> None:
    _check("gdn2_selftest_timeout", lib().gdn2_selftest_timeout(int(limit_cycles), _stream(stream)))


def gdn2_kernel_launches() -> int:
    return int(lib().gdn2_kernel_launches())


def gdn2_set_kernel_timer(enable: bool) -> None:
    lib().gdn2_set_kernel_timer(int(enable))


def gdn2_kernel_times() -> Dict[str, tuple]:
    """{kernel name: (launches, total ms)} for the kernels timed since the
    timer was enabled (only kinds that launched)."""
    n = lib().gdn2_kernel_kinds()
    counts = (ctypes.c_ulonglong * n)()
    ms = (ctypes.c_double * n)()
    _check("gdn2_kernel_times", lib().gdn2_kernel_times(ctypes.cast(counts, ctypes.c_void_p),
                                                         ctypes.cast(ms, ctypes.c_void_p), n))
    return {lib().gdn2_kernel_name(i).decode(): (counts[i], ms[i]) for i in range(n) if counts[i]}


# ------------------------------------------------------- tensor conveniences

def workspace(B, T, H, d_k, d_v, chunk, io, for_bwd, device="cuda") -> torch.Tensor:
    n = gdn2_workspace_bytes(B, T, H, d_k, d_v, chunk, io, for_bwd)
    if n == 0:
        raise Gdn2Error("gdn2_workspace_bytes", 2)
    return torch.empty(n, dtype=torch.uint8, device=device)


def check_device_status(stream=None) -> None:
    """Raise Gdn2Error if a kernel recorded an error (a bounded wait that gave
    up, or an operand outside the tensor-core path's fp16 range) since the
    status word was last read.  Waits for `stream`."""
    st = gdn2_get_device_status(stream)
    if st != 0:
        raise Gdn2Error("device status", st)


def _alloc_ws(n: int, fn: str, device) -> torch.Tensor:
    if n == 0:
        raise Gdn2Error(fn, 2)
    return torch.empty(n, dtype=torch.uint8, device=device)


def forward(q, k, v, g, b, w, S0=None, *, chunk: int = 64, want_state: bool = True,
            ws: Optional[torch.Tensor] = None, for_bwd: bool = False, stream=None,
            check: bool = True, gates: str = "activated"):
    """Returns (o, S_T or None, ws).  Shapes: q, k, g, b [B,T,H,dk]; v, w [B,T,H_v,dv]
    (H_v a multiple of H: grouped value heads); S0, S_T [B,H_v,dk,dv].  g, b, w
    may be bfloat16 (all three) on the tensor-core path.

    check=True (the default) waits for the stream and raises Gdn2Error if a
    kernel recorded an error during the call; check=False leaves the call
    asynchronous (read the status later with check_device_status)."""
    B, T, H, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    io, gio = _io_of(q), _gate_io_of(g, b, w, gates)
    if ws is None:
        ws = _alloc_ws(gdn2_workspace_bytes_ex(B, T, H, Hv, dk, dv, chunk, io, gio, for_bwd),
                       "gdn2_workspace_bytes_ex", q.device)
    o = torch.empty(B, T, Hv, dv, dtype=q.dtype, device=q.device)
    ST = torch.empty(B, Hv, dk, dv, dtype=torch.float32, device=q.device) if want_state else None
    gdn2_fwd_ex(q, k, v, g, b, w, S0, o, ST, ws, ws.numel(), B, T, H, Hv, dk, dv, chunk, io, gio,
                stream)
    if check:
        check_device_status(stream)
    return o, ST, ws


def backward(q, k, v, g, b, w, S0, dO, dST=None, *, chunk: int = 64,
             ws: Optional[torch.Tensor] = None, ws_has_fwd: bool = False,
             want_dS0: bool = True, stream=None, check: bool = True,
             gates: str = "activated") -> Dict[str, torch.Tensor]:
    """Gradients dq, dk, dv, dg, db, dw, dS0 (None unless want_dS0); dg, db, dw
    take the gates' dtype (and are of the logits with gates="logits").  check
    as in forward()."""
    B, T, H, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    io, gio = _io_of(q), _gate_io_of(g, b, w, gates)
    if ws is None:
        ws = _alloc_ws(gdn2_workspace_bytes_ex(B, T, H, Hv, dk, dv, chunk, io, gio, True),
                       "gdn2_workspace_bytes_ex", q.device)
        ws_has_fwd = False
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.empty_like(g), db=torch.empty_like(b), dw=torch.empty_like(w))
    out["dS0"] = (torch.empty(B, Hv, dk, dv, dtype=torch.float32, device=q.device)
                  if want_dS0 else None)
    gdn2_bwd_ex(q, k, v, g, b, w, S0, dO, dST, out["dq"], out["dk"], out["dv"], out["dg"],
                out["db"], out["dw"], out["dS0"], ws, ws.numel(), ws_has_fwd, B, T, H, Hv, dk, dv,
                chunk, io, gio, stream)
    if check:
        check_device_status(stream)
    return out


def forward_varlen(q, k, v, g, b, w, cu_seqlens, S0=None, *, chunk: int = 64,
                   want_state: bool = True, ws: Optional[torch.Tensor] = None,
                   for_bwd: bool = False, stream=None, check: bool = True, gates: str = "activated"):
    """Packed sequences: q, k, g, b [1,T,H,dk]; v, w [1,T,H_v,dv]; cu_seqlens
    int32 [N+1] on the device; S0 [N,H_v,dk,dv] or None.  Returns (o, S_T
    [N,...] or None, ws)."""
    _, T, H, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = cu_seqlens.numel() - 1
    io, gio = _io_of(q), _gate_io_of(g, b, w, gates)
    if ws is None:
        ws = _alloc_ws(gdn2_workspace_bytes_varlen(N, T, H, Hv, dk, dv, chunk, io, gio, for_bwd),
                       "gdn2_workspace_bytes_varlen", q.device)
    o = torch.empty(1, T, Hv, dv, dtype=q.dtype, device=q.device)
    ST = torch.empty(N, Hv, dk, dv, dtype=torch.float32, device=q.device) if want_state else None
    gdn2_fwd_varlen(q, k, v, g, b, w, S0, o, ST, ws, ws.numel(), cu_seqlens, N, T, H, Hv, dk, dv,
                    chunk, io, gio, stream)
    if check:
        check_device_status(stream)
    return o, ST, ws


def backward_varlen(q, k, v, g, b, w, cu_seqlens, S0, dO, dST=None, *, chunk: int = 64,
                    ws: Optional[torch.Tensor] = None, ws_has_fwd: bool = False,
                    want_dS0: bool = True, stream=None, check: bool = True,
                    gates: str = "activated") -> Dict[str, torch.Tensor]:
    """Gradients of forward_varlen: dq, dk, dv, dg, db, dw and dS0 [N,...]."""
    _, T, H, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = cu_seqlens.numel() - 1
    io, gio = _io_of(q), _gate_io_of(g, b, w, gates)
    if ws is None:
        ws = _alloc_ws(gdn2_workspace_bytes_varlen(N, T, H, Hv, dk, dv, chunk, io, gio, True),
                       "gdn2_workspace_bytes_varlen", q.device)
        ws_has_fwd = False
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.empty_like(g), db=torch.empty_like(b), dw=torch.empty_like(w))
    out["dS0"] = (torch.empty(N, Hv, dk, dv, dtype=torch.float32, device=q.device)
                  if want_dS0 else None)
    gdn2_bwd_varlen(q, k, v, g, b, w, S0, dO, dST, out["dq"], out["dk"], out["dv"], out["dg"],
                    out["db"], out["dw"], out["dS0"], ws, ws.numel(), ws_has_fwd, cu_seqlens, N, T,
                    H, Hv, dk, dv, chunk, io, gio, stream)
    if check:
        check_device_status(stream)
    return out


def decode_step(q, k, v, g, b, w, S, o=None, stream=None, gates: str = "activated"):
    """One token for N sequences: q, k, g, b [N,H,dk]; v, w [N,H_v,dv]; S
    [N,H_v,dk,dv] float32, updated in place.  Returns o [N,H_v,dv]."""
    N, H, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if o is None:
        o = torch.empty(N, Hv, dv, dtype=q.dtype, device=q.device)
    gdn2_decode_step_ex(q, k, v, g, b, w, S, o, N, H, Hv, dk, dv, _io_of(q), _gate_io_of(g, b, w, gates),
                        stream)
    return o
