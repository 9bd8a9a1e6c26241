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
