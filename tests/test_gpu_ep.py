"""Expert-parallel layer with R ranks emulated on one GPU, rows moved either by the library's put
kernels (expert-major receive buffers) or the way an all-to-all-v moves them (source-major,
one GEMM segment per source rank and local expert): the output of every rank against the layer
oracle over the whole batch (capacity counted over all ranks), and bit for bit against the
token-sharded layer that holds all experts on every rank."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _util import assert_layer_close, bf16_bits, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import moe_layer_router_b200 as m
    assert torch.cuda.is_available()
    return m


# (R, T per rank, d, E, k, f, f_shared, cap_mode, cf, zipf)
CASES = {
    "r2": (2, 96, 256, 8, 2, 192, 0, synth.CAP_NONE, 1.0, 0.0),
    "r4_shared_cap": (4, 64, 256, 16, 4, 128, 128, synth.CAP_PER_TOKEN, 1.25, 1.2),
    "r4_decode": (4, 8, 448, 32, 8, 192, 0, synth.CAP_NONE, 1.0, 0.0),
    "r2_pair_tiles": (2, 1024, 256, 4, 2, 256, 0, synth.CAP_PER_ASSIGNMENT, 1.1, 0.8),
}


@pytest.mark.parametrize("exchange", ["put", "fused", "a2a"])
@pytest.mark.parametrize("case", list(CASES))
def test_emulated_expert_parallel_layer(moe, case, exchange):
    from moe_layer_router_b200.ep import EmulatedEP
    R, T, d, E, k, f, fs, cap_mode, cf, zs = CASES[case]
    wl = synth.Workload("ep_" + case, R * T, d, E, k, f, f_shared=fs, cap_mode=cap_mode, capacity_factor=cf,
                        zipf_s=zs, seed=3)
    inp = synth.Inputs(wl)
    x = inp.x()
    wg = inp.wg()
    W1, W3, W2 = inp.w1(), inp.w3(), inp.w2()
    sh = [inp.shared(n) for n in ("w1s", "w3s", "w2s")] if fs else [None] * 3
    dv = to_dev_bf16
    dW1, dW3, dW2, dwg = dv(W1), dv(W3), dv(W2), dv(wg)
    dsh = [dv(a) if a is not None else None for a in sh]
    xs = [dv(x[r * T:(r + 1) * T]) for r in range(R)]
    outs = [torch.empty((T, d), dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    ep = EmulatedEP(R, T, d, E, k, f, fs, exchange=exchange)
    ep.forward(xs, dwg, None, dW1, dW3, dW2, *dsh, cf, cap_mode, outs)
    assert moe.moe_get_error() == 0

    # the token-sharded layer, all experts on every rank, same global capacity
    C = moe.moe_capacity(R * T, E, k, cf, cap_mode)
    wss = [torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
           for _ in range(R)]
    L = moe.moe_workspace_layout(T, d, E, k, f, fs)
    for r in range(R):
        moe.moe_layer_route_count(xs[r], dwg, None, fs, T, d, E, k, f, wss[r])
    allc = torch.stack([moe.workspace_view(wss[r], L, "counts_raw", (E,), torch.int32) for r in range(R)])
    outs_dp = []
    for r in range(R):
        fb = torch.empty(E, dtype=torch.int32, device="cuda")
        moe.moe_fill_base(allc, R, r, E, fb)
        o = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        moe.moe_layer_finish(xs[r], dW1, dW3, dW2, *dsh, fs, T, d, E, k, f, C, fb, o, wss[r])
        outs_dp.append(o)
    assert moe.moe_get_error() == 0

    # oracle over the whole batch, routing the GPU's logits
    logits = np.concatenate([moe.workspace_view(b.ws, b.layout, "logits", (T, E), torch.float32).cpu().numpy()
                             for b in ep.ranks])
    ref = oracle.layer_forward(x, wg, W1, W3, W2, k=k, C=C, logits_in=logits, W1s=sh[0], W3s=sh[1], W2s=sh[2])
    got = np.concatenate([bf16_bits(o) for o in outs])
    assert_layer_close(got, ref["out"], "expert-parallel layer")
    # every rank kept exactly the rows the whole-batch dispatch keeps
    kept = sum(int(moe.workspace_view(b.ws, b.layout, "counts", (E,), torch.int32).sum()) for b in ep.ranks)
    assert kept == ref["N"]
    if cap_mode != synth.CAP_NONE:
        assert kept < R * T * k          # capacity dropped rows
    # tile kind: pair (2-SM) tiles when the rows per expert average >= 256 (local experts for EP)
    same_tiles = (R * T * k >= 256 * (E // R)) == (T * k >= 256 * E)
    if same_tiles:   # same tile kind in both paths: each row's arithmetic is the same
        for r in range(R):
            assert torch.equal(outs[r].view(torch.int16), outs_dp[r].view(torch.int16)), f"rank {r}"


def test_nccl_driver_single_rank_matches_layer(moe):
    """ep_layer_forward_dist on one NCCL rank (the all-gather and both all_to_all_single calls run,
    rows arrive source-major, the GEMMs run the source-major segments): bit-identical to the
    single-GPU layer."""
    import os
    import socket
    import torch.distributed as dist
    from moe_layer_router_b200.ep import ep_layer_forward_dist
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = synth.Workload("ep_nccl", 64, 256, 8, 2, 128, f_shared=128, cap_mode=synth.CAP_PER_TOKEN,
                            capacity_factor=1.0, seed=5)
        inp = synth.Inputs(wl)
        T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
        dv = to_dev_bf16
        x, wg = dv(inp.x()), dv(inp.wg())
        W1, W3, W2 = dv(inp.w1()), dv(inp.w3()), dv(inp.w2())
        sh = [dv(inp.shared(n)) for n in ("w1s", "w3s", "w2s")]
        out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        ep_layer_forward_dist(x, wg, None, W1, W3, W2, *sh, fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode, out)
        ref = torch.empty_like(out)
        ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
        moe.moe_layer_forward(x, wg, None, W1, W3, W2, *sh, fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode,
                              ref, ws)
        torch.cuda.synchronize()
        assert moe.moe_get_error() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    finally:
        dist.destroy_process_group()


def test_plan_split_table_matches_host_reference(moe):
    """moe_ep_plan's [2, R] split table (the all-to-all-v split sizes) against the host restatement
    of the whole-batch capacity over ranks, for every rank of a skewed batch with capacity."""
    from _ep_reference import ep_row_splits
    R, E = 4, 32
    rng = np.random.default_rng(5)
    counts = rng.integers(0, 60, size=(R, E)).astype(np.int32)
    counts[:, :3] += 100                                   # hot experts, so the capacity bites
    for C in (-1, 0, 70, 150):
        dev_counts = torch.from_numpy(counts).cuda()
        for r in range(R):
            ep_ws = torch.empty(moe.moe_ep_workspace_bytes(R, E), dtype=torch.uint8, device="cuda")
            moe.moe_ep_plan(dev_counts, R, r, E, C, R * 512, ep_ws)
            got = moe.moe_ep_splits(ep_ws, R, E).cpu().tolist()
            send, recv = ep_row_splits(counts, C, r)
            assert got == [send, recv], (C, r)
    assert moe.moe_get_error() == 0


def test_put_driver_single_rank_matches_layer(moe):
    """ep_layer_forward_put_dist on one NCCL rank (its own buffers, no IPC import; the barriers and
    the expert-major put path run): bit-identical to the single-GPU layer."""
    import os
    import socket
    import torch.distributed as dist
    from moe_layer_router_b200.ep import PeerBuffers, _RankBuffers, ep_layer_forward_put_dist
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = synth.Workload("ep_put", 96, 256, 8, 2, 128, f_shared=128, cap_mode=synth.CAP_PER_TOKEN,
                            capacity_factor=1.0, seed=6)
        inp = synth.Inputs(wl)
        T, d, E, k, f, fs = wl.T, wl.d, wl.E, wl.k, wl.f, wl.f_shared
        dv = to_dev_bf16
        x, wg = dv(inp.x()), dv(inp.wg())
        W1, W3, W2 = dv(inp.w1()), dv(inp.w3()), dv(inp.w2())
        sh = [dv(inp.shared(n)) for n in ("w1s", "w3s", "w2s")]
        bufs = _RankBuffers(moe, 1, T, d, E, k, f, fs, T * k, x.device)
        peers = PeerBuffers(bufs.recv, bufs.view(moe, "y_perm", (T * k, d), torch.bfloat16))
        out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        for _ in range(2):                       # a second call reuses the buffers
            ep_layer_forward_put_dist(x, wg, None, W1, W3, W2, *sh, fs, T, d, E, k, f, wl.capacity_factor,
                                      wl.cap_mode, out, bufs, peers)
        peers.close()
        ref = torch.empty_like(out)
        ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device="cuda")
        moe.moe_layer_forward(x, wg, None, W1, W3, W2, *sh, fs, T, d, E, k, f, wl.capacity_factor, wl.cap_mode,
                              ref, ws)
        torch.cuda.synchronize()
        assert moe.moe_get_error() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    finally:
        dist.destroy_process_group()


def _ipc_child(handle, rows, d, E, q):
    """Imports the parent's receive buffer and puts its rows there with the dispatch kernel (R = 1:
    the whole x_perm goes to rank 0's buffer, expert-major = x_perm order)."""
    try:
        import torch
        import moe_layer_router_b200 as moe
        torch.cuda.set_device(0)
        x_perm = to_dev_bf16(synth.normal_bf16(9, 1, 0, rows * d, 1.0).reshape(rows, d))
        counts = np.full((1, E), rows // E, np.int32)
        ep_ws = torch.empty(moe.moe_ep_workspace_bytes(1, E), dtype=torch.uint8, device="cuda")
        moe.moe_ep_plan(torch.from_numpy(counts).cuda(), 1, 0, E, -1, rows, ep_ws)
        addr = moe.moe_ipc_import(handle)
        moe.moe_ep_dispatch(x_perm, 1, 0, E, d, [addr], ep_ws)
        torch.cuda.synchronize()
        rc = moe.moe_get_error()
        moe.moe_ipc_close(addr, handle)
        q.put(("ok", rc))
    except Exception as e:      # reported to the parent, which fails the test
        q.put(("error", repr(e)))


def test_ipc_peer_put_from_another_process(moe):
    """A second process on the same GPU imports this process's receive buffer (moe_ipc_export /
    moe_ipc_import) and the library's put kernel stores rows into it: the rows arrive intact, at the
    exported pointer's offset inside its allocation."""
    import subprocess
    import torch.multiprocessing as mp
    mode = subprocess.run(["nvidia-smi", "--query-gpu=compute_mode", "--format=csv,noheader", "-i", "0"],
                          capture_output=True, text=True).stdout.strip()
    if "Exclusive" in mode:
        pytest.skip(f"compute mode {mode}: a second process cannot use the GPU")
    rows, d, E = 512, 256, 4
    pad = torch.zeros(4096, dtype=torch.uint8, device="cuda")        # an allocation with an offset inside
    recv = torch.zeros((rows + 8, d), dtype=torch.bfloat16, device="cuda")
    handle = moe.moe_ipc_export(recv[8:])
    assert len(handle) == moe.MOE_IPC_HANDLE_BYTES
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_ipc_child, args=(handle, rows, d, E, q))
    p.start()
    status, info = q.get(timeout=300)
    p.join(timeout=120)
    assert status == "ok" and info == 0, info
    assert p.exitcode == 0
    want = synth.normal_bf16(9, 1, 0, rows * d, 1.0).reshape(rows, d)
    assert np.array_equal(bf16_bits(recv[8:]), want)
    assert not bf16_bits(recv[:8]).any()                  # nothing before the exported pointer
    del pad
