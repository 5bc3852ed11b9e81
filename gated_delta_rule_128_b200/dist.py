"""Multi-GPU plumbing for running the operator on N GPUs of one node.

The operator's (batch, head) pairs are independent problems, so N GPUs need
no data-path collective: every rank runs its own batch (weak scaling), and
the ranks only meet at barriers and to take the slowest rank's time.  One
process per GPU, launched by torchrun (RANK / LOCAL_RANK / WORLD_SIZE /
MASTER_ADDR / MASTER_PORT in the environment); NCCL on GPUs, gloo on CPU.
"""

from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import List

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, info: RankInfo, timeout_s: int = 120) -> None:
    """Join the process group when there is more than one rank."""
    if info.world <= 1 or dist.is_initialized():
        return
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if backend == "nccl":
        torch.cuda.set_device(info.local_rank)
        kw["device_id"] = torch.device("cuda", info.local_rank)
    dist.init_process_group(backend, **kw)


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(values: List[float], device=None) -> List[float]:
    """Element-wise maximum of `values` over all ranks (identity on one rank)."""
    if not dist.is_initialized():
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: rank 0 keeps the workload's own seed."""
    return base_seed + 7919 * rank


def batch_rows(total_rows: int, world: int, rank: int) -> range:
    """Contiguous share of `total_rows` batch rows for `rank` (for strong
    scaling of one fixed batch; earlier ranks take the remainder)."""
    base, extra = divmod(total_rows, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
