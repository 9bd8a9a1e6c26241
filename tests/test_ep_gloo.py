"""Expert-parallel host logic on CPU: the kept counts and row splits against brute force over the
whole batch, and the all-to-all-v row exchange among gloo ranks (world size 2 and 3): received
rows arrive in (source rank, local expert) order and results come back to the rows they left."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from _ep_reference import ep_row_splits, kept_counts
from moe_layer_router_b200.ep import exchange_rows


def _batch(R, T, E, k, seed):
    rng = np.random.default_rng(seed)
    # skewed routes so that capacity bites on the popular experts
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    p /= p.sum()
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(R * T)]).astype(np.int32)
    return idx


def _kept_brute(idx, R, T, E, C):
    """Rows of each rank kept per expert, by walking the whole batch's assignments in token order."""
    taken = np.zeros(E, np.int64)
    kept = np.zeros((R, E), np.int64)
    for t in range(idx.shape[0]):
        for e in idx[t]:
            if C < 0 or taken[e] < C:
                kept[t // T, e] += 1
            taken[e] += 1
    return kept


@pytest.mark.parametrize("R,T,E,k,C", [(2, 64, 8, 2, -1), (2, 64, 8, 2, 12), (4, 32, 16, 4, 5), (3, 50, 12, 3, 0),
                                       (8, 16, 64, 8, 2)])
def test_kept_counts_and_splits_match_brute_force(R, T, E, k, C):
    idx = _batch(R, T, E, k, seed=R * 100 + E)
    counts_raw = np.stack([np.bincount(idx[r * T:(r + 1) * T].ravel(), minlength=E) for r in range(R)])
    want = _kept_brute(idx, R, T, E, C)
    assert np.array_equal(kept_counts(counts_raw, C), want)
    # the oracle's whole-batch dispatch keeps the same number of rows per expert
    d = oracle.dispatch(idx, E, C)
    assert np.array_equal(want.sum(axis=0), d["counts"])
    El = E // R
    for r in range(R):
        send, recv = ep_row_splits(counts_raw, C, r)
        assert send == [int(want[r, q * El:(q + 1) * El].sum()) for q in range(R)]
        assert recv == [int(want[s, r * El:(r + 1) * El].sum()) for s in range(R)]


def _x_perm(idx, R, T, E, C, rank, d):
    """Rank `rank`'s kept rows in expert order (token order inside an expert), as float rows that
    encode (token, expert), plus the expert of each row."""
    taken = np.zeros(E, np.int64)
    rows = []
    for t in range(idx.shape[0]):
        for e in idx[t]:
            keep = C < 0 or taken[e] < C
            taken[e] += 1
            if keep and t // T == rank:
                rows.append((e, t))
    rows.sort(key=lambda r: (r[0], r[1]))    # stable: token order within an expert
    x = np.zeros((max(len(rows), 1), d), np.float32)
    for i, (e, t) in enumerate(rows):
        x[i] = t * 1000.0 + e + np.arange(d) * 100000.0     # integers: exact in float32
    return x[:len(rows)], np.array([e for e, _ in rows], np.int64)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, R, port, T, E, k, C, d, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        idx = _batch(R, T, E, k, seed=7)
        counts_raw = np.stack([np.bincount(idx[r * T:(r + 1) * T].ravel(), minlength=E) for r in range(R)])
        # what every rank learns from the all-gather of raw counts
        mine = torch.from_numpy(counts_raw[rank].astype(np.int32))
        gathered = [torch.empty(E, dtype=torch.int32) for _ in range(R)]
        dist.all_gather(gathered, mine)
        all_counts = torch.stack(gathered).numpy()
        assert np.array_equal(all_counts, counts_raw)
        send, recv = ep_row_splits(all_counts, C, rank)
        x, ex = _x_perm(idx, R, T, E, C, rank, d)
        xt = torch.from_numpy(np.ascontiguousarray(x)) if len(x) else torch.zeros((0, d))
        out = torch.zeros((R * T * k, d))
        exchange_rows(xt, send, recv, out)
        got = out[:sum(recv)].numpy()
        # expected receive layout: for each source s, its kept rows of my experts, expert-major
        El = E // R
        want = []
        for s in range(R):
            xs, es = _x_perm(idx, R, T, E, C, s, d)
            sel = (es >= rank * El) & (es < (rank + 1) * El)
            want.append(xs[sel])
        want = np.concatenate(want) if want else np.zeros((0, d), np.float32)
        ok_recv = np.array_equal(got, want)
        # "experts": y = 2 x + expert id of the row (read back from the row's encoding)
        e_of = np.rint(got[:, 0] % 1000.0).astype(np.float32) if len(got) else np.zeros(0, np.float32)
        y = torch.from_numpy(np.ascontiguousarray(2 * got + e_of[:, None], dtype=np.float32)) if len(got) \
            else torch.zeros((0, d))
        back = torch.zeros((T * k, d))
        exchange_rows(y, recv, send, back)
        want_back = (2 * x + ex[:, None].astype(np.float32)).astype(np.float32)
        ok_back = np.array_equal(back[:sum(send)].numpy(), want_back) if len(x) else sum(send) == 0
        q.put((rank, bool(ok_recv), bool(ok_back), sum(recv)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R,C", [(2, -1), (3, 6)])
def test_all_to_all_v_exchange_between_gloo_ranks(R, C):
    T, E, k, d = 24, 6 * R, 2, 8
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, R, port, T, E, k, C, d, q)) for r in range(R)]
    for p in procs:
        p.start()
    res = []
    for _ in range(R):
        res.append(q.get(timeout=120))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_recv, ok_back, n in sorted(res):
        assert ok_recv, f"rank {rank}: received rows out of (source, expert) order"
        assert ok_back, f"rank {rank}: results did not come back to their rows"
    assert sum(n for *_, n in res) > 0


def _peer_worker(rank, R, port, q):
    """PeerBuffers on gloo ranks with stand-in export / import / close: every rank ends up with its
    own buffers at its own index and the other ranks' imported addresses, in rank order, and
    closes exactly what it imported."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        from moe_layer_router_b200.ep import PeerBuffers
        opened, closed = [], []

        def export(buf):
            return f"{rank}:{buf}".encode()

        def import_(h):
            s, name = h.decode().split(":")
            a = 1000 * int(s) + (1 if name == "recv" else 2)
            opened.append(a)
            return a

        def close(a, h):
            assert import_(h) == a
            closed.append(a)

        pb = PeerBuffers("recv", "y_perm", export=export, import_=import_, close=close)
        ok = pb.recv[rank] == "recv" and pb.y_perm[rank] == "y_perm"
        ok &= all(pb.recv[s] == 1000 * s + 1 and pb.y_perm[s] == 1000 * s + 2 for s in range(R) if s != rank)
        ok &= len(opened) == 2 * (R - 1)
        n_open = len(opened)
        pb.close()
        ok &= sorted(closed) == sorted(opened[:n_open]) and not pb._opened
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R", [2, 3])
def test_peer_buffer_handle_exchange_between_gloo_ranks(R):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_worker, args=(r, R, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(R)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok in res), res
