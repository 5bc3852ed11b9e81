"""Helpers shared by the tests: tolerance metric and input marshalling."""

from typing import Dict

import numpy as np
import torch

from gated_delta_rule_128_b200 import workloads

TOL_F32 = 1e-4        # float32 path: max|err| / max|ref|
TOL_BF16_OUT = 5e-3   # bf16-I/O path: o and S_T
TOL_BF16_GRAD = 1e-2  # bf16-I/O path: gradients

IO_NAMES = ("q", "k", "v", "dO")   # tensors carried in the io type
GATE_NAMES = ("g", "b", "w")       # tensors carried in the gate type


def rel(a, ref) -> float:
    """max|a - ref| / max|ref| over one output tensor (the pages' tolerance
    is stated per output; a zero reference falls back to absolute error)."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(a - ref)) / (den if den > 0 else 1.0)) if ref.size else 0.0


def io_round(x: Dict[str, torch.Tensor], io: str, gates: str = "f32") -> Dict[str, torch.Tensor]:
    """The float32 values each side consumes: bf16-I/O rounds q, k, v, dO, and
    bf16 gates round g, b, w."""
    names = (IO_NAMES if io == "bf16" else ()) + (GATE_NAMES if gates == "bf16" else ())
    return {n: (workloads.round_bf16(t) if n in names else t) for n, t in x.items()}


def to_np64(x: Dict[str, torch.Tensor]) -> Dict[str, np.ndarray]:
    return {n: t.double().numpy() for n, t in x.items()}


def to_device(x: Dict[str, torch.Tensor], io: str, device="cuda",
              gates: str = "f32") -> Dict[str, torch.Tensor]:
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    gt = torch.bfloat16 if gates == "bf16" else torch.float32
    return {n: (t.to(dt) if n in IO_NAMES else t.to(gt) if n in GATE_NAMES else t).contiguous().to(device)
            for n, t in x.items()}
