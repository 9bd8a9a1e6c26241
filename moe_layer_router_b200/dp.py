"""Data-parallel plumbing for the MoE layer forward: one process per GPU.

The layer is per token ([EP-KV] §4: a token's MLP/MoE output never reads another token's;
§2: each token is routed on its own), so the data-parallel path gives each rank
its own token batch against replicated weights and needs no collective on the data path.
What remains is host logic: which token rows a rank owns, and how a timing over ranks is
combined (the slowest rank bounds the job).  It works on any torch.distributed backend
(NCCL on GPUs, gloo on CPU for tests).

The one exchange: when ONE global batch is split over ranks and a capacity limit applies,
token-order dropping is global ([EP-DS3] §2.1 capacity; the oracle's reading: the first C
assignments of each expert in token order are kept).  Rank r must then know how many
assignments of each expert the tokens of ranks 0..r-1 made: an all-gather of the per-expert
counts [G, E] and a prefix over ranks (sharded_layer_forward).
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


def fill_base_host(all_counts, rank: int):
    """Host form of the rank prefix: sum of rows < rank of a [G, E] count table."""
    import numpy as np
    a = np.asarray(all_counts, dtype=np.int64)
    return a[:rank].sum(axis=0).astype(np.int32) if rank > 0 else np.zeros(a.shape[1], np.int32)


def sharded_layer_forward(moe, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity,
                          out, ws, fill_base, all_counts, group=None, stream=None) -> None:
    """One rank's share of a global batch with a global token-order capacity.

    moe_layer_route_count -> all-gather of counts_raw into all_counts [G, E] (int32, device)
    -> moe_fill_base -> moe_layer_finish.  `capacity` is the global batch's (moe_capacity of
    the global token count); fill_base [E] and all_counts [G, E] are caller-owned int32.
    """
    import torch.distributed as dist
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    moe.moe_layer_route_count(x, Wg, bias, f_shared, T, d, E, k, f, ws, stream)
    layout = moe.moe_workspace_layout(T, d, E, k, f, f_shared)
    import torch
    counts = moe.workspace_view(ws, layout, "counts_raw", (E,), torch.int32)
    if G > 1:
        dist.all_gather_into_tensor(all_counts.view(-1), counts, group=group)
    moe.moe_fill_base(all_counts, G, rank, E, fill_base, stream)      # rank 0 (or G = 1): zeros
    moe.moe_layer_finish(x, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity, fill_base, out, ws, stream)

