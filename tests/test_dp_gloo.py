"""The multi-process (N > 1) host path on CPU: world_size-2 gloo ranks.

Covers what bench.py's torchrun path does besides the kernels: each rank owns its own
token rows (distinct, contiguous), the timed region is reduced to the slowest rank, and
the whole-job throughput counts every rank's tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    from moe_layer_router_b200 import dp
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T = 64
        row0, n = dp.token_rows(rank, world, T)
        inp = synth.Inputs(synth.WORKLOADS["tiny"])
        x = inp.x_rows(row0, n)
        # every rank's rows, gathered: distinct and equal to the generator's global rows
        xs = [torch.zeros(n * 256, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(xs, torch.from_numpy(x.astype(np.int32)))         # gloo has no 16-bit ints
        whole = np.concatenate([t.numpy().astype(np.uint16) for t in xs])
        ok_rows = np.array_equal(whole, inp.x_rows(0, world * T))
        local_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        mx = dp.max_over_ranks(local_ms)
        val = dp.job_throughput(T, world, 7, mx)
        s0, c0 = dp.split_rows(101, rank, world)
        sizes = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([s0, c0]))
        out[rank] = (ok_rows, mx, val, [tuple(t.tolist()) for t in sizes])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_rows_timing_and_throughput():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        ok_rows, mx, val, sizes = out[r]
        assert ok_rows
        assert mx == 15.0                                  # the slowest rank's time
        assert val == pytest.approx(world * 64 * 7 / 0.015)
        assert sizes == [(0, 51), (51, 50)]                # contiguous, covering 101 rows


def test_single_process_helpers():
    from moe_layer_router_b200 import dp
    assert dp.token_rows(3, 4, 100) == (300, 100)
    assert [dp.split_rows(10, r, 3) for r in range(3)] == [(0, 4), (4, 3), (7, 3)]
    assert dp.max_over_ranks(2.5) == 2.5
    assert dp.job_throughput(4096, 8, 10, 20.0) == pytest.approx(8 * 4096 * 10 / 0.02)
    with pytest.raises(ValueError):
        dp.token_rows(2, 2, 10)


def _capacity_worker(rank, world, port, out):
    """Each rank holds one shard of a global routing; the exchange of per-expert counts must
    reproduce the global token-order capacity of the oracle on the whole batch."""
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from moe_layer_router_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, E, k = 500, 12, 2
        rng = np.random.default_rng(5)
        logits = (rng.standard_normal((T * world, E)) + np.linspace(2, -2, E)).astype(np.float32)
        idx, _ = oracle.route(logits, k)
        C = oracle.capacity(T * world, E, k, 0.8, oracle.CAP_PER_ASSIGNMENT)
        glob = oracle.dispatch(idx, E, C)
        mine = idx[rank * T:(rank + 1) * T]
        local = oracle.dispatch(mine, E, -1)["counts_raw"]
        table = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(table, torch.from_numpy(local))
        base = dp.fill_base_host(torch.stack(table).numpy(), rank)
        # keep rule of one shard: position of the assignment among this shard's assignments to
        # its expert, in token order, plus the base, below C
        kept = np.zeros_like(mine, dtype=bool)
        pos = np.zeros(E, np.int64)
        for t in range(T):
            for j in range(k):
                e = mine[t, j]
                kept[t, j] = base[e] + pos[e] < C
                pos[e] += 1
        want = glob["dest"][rank * T:(rank + 1) * T] >= 0
        out[rank] = (bool(np.array_equal(kept, want)), int(kept.sum()), int(glob["N"]),
                     bool((glob["counts_raw"] > C).any()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_global_capacity_exchange():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_capacity_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert all(out[r][0] for r in range(world))
    assert out[0][1] + out[1][1] == out[0][2]          # kept over ranks = kept of the whole batch
    assert out[0][3]                                   # the capacity did bind


def test_fill_base_host():
    from moe_layer_router_b200 import dp
    t = np.array([[1, 2, 3], [4, 5, 6], [7, 8, 9]], np.int32)
    assert list(dp.fill_base_host(t, 0)) == [0, 0, 0]
    assert list(dp.fill_base_host(t, 2)) == [5, 7, 9]
