"""Seeded synthetic inputs for the Gated Delta Rule-2 operator.

This module only draws random tensors.  It holds none of the operator's
arithmetic, so both the CUDA path and the fp64 oracle can be fed from it.

Recipe (the same for every workload; the pages name no operator benchmark, so
these synthetic tensors stand in for the FineWeb-Edu activations of the
"Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention" pages):

* A CPU ``torch.Generator`` seeded with ``1000 + workload index``.
* Tensors drawn in float32 in the fixed order q, k, v, g, b, w, S0, dO.
* q, k ~ N(0, 1), then L2-normalised over the key axis per token and head.
* v ~ N(0, 1).
* erase gate b = sigmoid(N(0, 1)), or 2 * sigmoid(N(0, 1)) where the erase
  range is widened to [0, 2] (negative eigenvalues).
* write gate w = sigmoid(N(0, 1)).
* log-decay g = logsigmoid(N(0, 1)) / 16 per key channel.
* S0 = 0, or N(0, 0.02^2) (standard deviation 0.02).
* dO ~ N(0, 1).

Tied variants reproduce the special cases named on the pages: KDA ties
b = w = beta * 1 with beta = sigmoid(N(0, 1)) per token and head; Gated
DeltaNet additionally ties the decay to one scalar per token and head.

Decode: the state S0 comes from a generator seeded with the workload seed; the
inputs of step s come from a generator seeded with ``seed * 1_000_003 + s``, so
that any single step can be drawn on its own.

Layouts: activations and gates are [B, T, H, D] (D fastest); the state is
[B, H, d_k, d_v] (d_v fastest).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    io: str            # "f32" or "bf16": dtype of q, k, v, o, dO, dq, dk, dv
    backward: bool     # whether the workload runs gdn2_bwd
    s0_std: float      # 0.0 => S0 = 0
    erase_scale: float = 1.0   # b = erase_scale * sigmoid(N(0,1))
    decode_steps: int = 0      # > 0 => a recurrent-decode workload (T is 1)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H


WORKLOADS: Dict[int, Workload] = {
    0: Workload(0, "tiny-fp32-fwd-bwd B1 T256 H2 d32 C64", 1, 256, 2, 32, 32, 64,
                "f32", True, 0.0),
    1: Workload(1, "fwd B8 T2048 H16 d128 C64 bf16", 8, 2048, 16, 128, 128, 64,
                "bf16", False, 0.02),
    2: Workload(2, "fwd+bwd B4 T4096 H16 d128 C64 bf16", 4, 4096, 16, 128, 128, 64,
                "bf16", True, 0.0),
    3: Workload(3, "fwd+bwd long B1 T16384 H16 d128 C64 bf16 b in [0,2]", 1, 16384, 16,
                128, 128, 64, "bf16", True, 0.0, erase_scale=2.0),
    4: Workload(4, "decode N256 H16 d128 x1024 steps bf16", 256, 1, 16, 128, 128, 64,
                "bf16", False, 0.02, decode_steps=1024),
}


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def draw(B: int, T: int, H: int, dk: int, dv: int, seed: int, *,
         s0_std: float = 0.0, erase_scale: float = 1.0, tie: Optional[str] = None,
         with_dO: bool = True, with_dST: bool = False) -> Dict[str, torch.Tensor]:
    """Draw one set of float32 CPU inputs.

    ``tie``: None (independent gates), "kda" (b = w = beta * 1) or "gdn"
    (b = w = beta * 1 and g = one scalar per token and head).  When tied, the
    per-token scalars are also returned as ``beta`` [B,T,H] and, for "gdn",
    ``alpha_log`` [B,T,H].
    """
    gen = torch.Generator().manual_seed(seed)
    f = dict(dtype=torch.float32, generator=gen)
    q = _l2norm(torch.randn(B, T, H, dk, **f))
    k = _l2norm(torch.randn(B, T, H, dk, **f))
    v = torch.randn(B, T, H, dv, **f)
    out: Dict[str, torch.Tensor] = {}
    if tie is None:
        g = torch.nn.functional.logsigmoid(torch.randn(B, T, H, dk, **f)) / 16
        b = erase_scale * torch.sigmoid(torch.randn(B, T, H, dk, **f))
        w = torch.sigmoid(torch.randn(B, T, H, dv, **f))
    elif tie in ("kda", "gdn"):
        if tie == "kda":
            g = torch.nn.functional.logsigmoid(torch.randn(B, T, H, dk, **f)) / 16
        else:
            a = torch.nn.functional.logsigmoid(torch.randn(B, T, H, 1, **f)) / 16
            g = a.expand(B, T, H, dk).contiguous()
            out["alpha_log"] = a[..., 0].contiguous()
        beta = torch.sigmoid(torch.randn(B, T, H, 1, **f))
        b = beta.expand(B, T, H, dk).contiguous()
        w = beta.expand(B, T, H, dv).contiguous()
        out["beta"] = beta[..., 0].contiguous()
    else:
        raise ValueError(f"unknown tie {tie!r}")
    if s0_std > 0:
        S0 = torch.randn(B, H, dk, dv, **f) * s0_std
    else:
        S0 = torch.zeros(B, H, dk, dv, dtype=torch.float32)
    out.update(q=q, k=k, v=v, g=g, b=b, w=w, S0=S0)
    if with_dO:
        out["dO"] = torch.randn(B, T, H, dv, **f)
    if with_dST:
        out["dST"] = torch.randn(B, H, dk, dv, **f)
    return out


def draw_workload(index: int, *, tie: Optional[str] = None, T: Optional[int] = None,
                  B: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Inputs of one of the five workloads (optionally with fewer tokens or batch
    rows, drawn from the same seed: a smaller problem of the same distribution)."""
    wl = WORKLOADS[index]
    return draw(B or wl.B, T or wl.T, wl.H, wl.dk, wl.dv, wl.seed, s0_std=wl.s0_std,
                erase_scale=wl.erase_scale, tie=tie, with_dO=wl.backward)


def round_bf16(x: torch.Tensor) -> torch.Tensor:
    """Round float32 values to bf16 and widen back: the values a bf16-I/O call
    consumes, which the oracle must consume too."""
    return x.to(torch.bfloat16).to(torch.float32)


def decode_state(N: int, H: int, dk: int, dv: int, seed: int, s0_std: float) -> torch.Tensor:
    gen = torch.Generator().manual_seed(seed)
    return torch.randn(N, H, dk, dv, dtype=torch.float32, generator=gen) * s0_std


def decode_step_inputs(N: int, H: int, dk: int, dv: int, seed: int, step: int,
                       erase_scale: float = 1.0) -> Dict[str, torch.Tensor]:
    """Inputs of one decode step, [N, H, D] each (T = 1 squeezed)."""
    d = draw(N, 1, H, dk, dv, seed * 1_000_003 + step, erase_scale=erase_scale,
             with_dO=False)
    return {n: d[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "b", "w")}


def packed_lengths(total: int, seed: int, lo: int = 1, hi: int = 2048) -> list:
    """Sequence lengths for a packed batch of `total` tokens: drawn uniformly
    from [lo, hi] (seeded) until they fill `total`, the last one cut to fit.
    A stand-in for documents of mixed lengths packed into one training row."""
    gen = torch.Generator().manual_seed(seed)
    lens, left = [], total
    while left > 0:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        lens.append(min(n, left))
        left -= lens[-1]
    return lens
