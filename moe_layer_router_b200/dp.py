"""Data-parallel plumbing for the MoE layer forward: one process per GPU.

The layer is per token ([EP-KV] §4: a token's MLP/MoE output never reads another token's;
§2: each token is routed on its own), so the data-parallel path gives each rank
its own token batch against replicated weights and needs no collective on the data path.
What remains is host logic: which token rows a rank owns, and how a timing over ranks is
combined (the slowest rank bounds the job).  It works on any torch.distributed backend
(NCCL on GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

from typing import Optional, Tuple


def token_rows(rank: int, world: int, T_per_rank: int) -> Tuple[int, int]:
    """First global row and row count of this rank's batch (weak scaling: T rows per rank)."""
    if not (0 <= rank < world) or T_per_rank < 1:
        raise ValueError("bad rank / world / batch")
    return rank * T_per_rank, T_per_rank


def split_rows(T_total: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous near-equal split of T_total rows (strong scaling): (first row, count)."""
    if not (0 <= rank < world) or T_total < 0:
        raise ValueError("bad rank / world / rows")
    base, extra = divmod(T_total, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None, device=None) -> float:
    """The largest `value` over the ranks of `group` (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("non-positive time")
    return world * tokens_per_rank * steps / (max_ms / 1000.0)


def env_rank() -> Tuple[int, int, int]:
    """(rank, world, local rank) from the torchrun environment (single process: 0, 1, 0)."""
    import os
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))
