"""Host reference for the expert-parallel split sizes (test helper).

The library computes these on the device (moe_ep_plan writes the [2, R] split table); this
module restates them on the host so that the CPU tests can drive an all-to-all-v between gloo
ranks and the GPU tests can check the device's table against them.
"""
import numpy as np


def kept_counts(all_counts_raw: np.ndarray, capacity: int) -> np.ndarray:
    """[R, E] rows each rank keeps per expert: the rows of rank r for expert e come after the
    rows of ranks < r in token order, so r keeps min(c[r][e], max(0, C - sum_{s<r} c[s][e]))."""
    c = np.asarray(all_counts_raw, dtype=np.int64)
    if capacity < 0:
        return c.copy()
    before = np.cumsum(c, axis=0) - c
    return np.clip(np.minimum(c, capacity - before), 0, None)


def ep_row_splits(all_counts_raw: np.ndarray, capacity: int, rank: int):
    """-> (send_rows [R], recv_rows [R]): rows `rank` sends to each rank (its kept rows of that
    rank's experts, in rank order = x_perm order) and rows it receives from each rank."""
    R, E = all_counts_raw.shape
    if E % R:
        raise ValueError("E must be a multiple of the number of ranks")
    El = E // R
    kept = kept_counts(all_counts_raw, capacity)
    per_rank = kept.reshape(R, R, El).sum(axis=2)       # [src, dst]
    return per_rank[rank].tolist(), per_rank[:, rank].tolist()
