"""Expert parallelism around the C ABI: experts split over R ranks.

Rank r holds the E / R experts [r El, (r + 1) El) (uniform contiguous split, [EP-DS3]
section 3.1 _assign_experts).  A layer call per rank: route and count its own tokens, all-gather
the raw counts [R, E], keep rows under the whole batch's capacity (token order over ranks in rank
order), send each kept row to its expert's rank, run the local experts over the received rows,
send the results back and combine ([EP-KV] sections 6-7).  Every step of the path runs in the
library's kernels; this module only moves pointers, sizes and (for the NCCL path) the two
all-to-all-v exchanges.

Three drivers:
  * ``EmulatedEP``: R ranks on one device in one process.  The row exchanges are the library's
    put kernels writing into the other ranks' buffers (expert-major receive order, one GEMM group
    per local expert); the all-gather is a device copy.
  * ``ep_layer_forward_dist``: one process per GPU over ``torch.distributed``; counts are
    all-gathered and rows moved with ``all_to_all_single`` (NCCL), whose split sizes the
    device-side plan writes (``moe_ep_splits``; the host only reads them back, as the collective
    wants them on the host); rows arrive source-major and the local GEMM runs one segment per
    (source rank, local expert).
  * ``ep_layer_forward_put_dist``: one process per GPU, rows moved by the library's put kernels
    straight into the other ranks' buffers (``PeerBuffers``: CUDA IPC handles exchanged over
    ``torch.distributed``), with a barrier between the puts and the reads of each exchange.
"""
from __future__ import annotations

from typing import List, Optional, Sequence


def exchange_rows(src, send_rows: Sequence[int], recv_rows: Sequence[int], out, group=None) -> None:
    """all_to_all_single over the leading (row) dimension: rows [sum(send[:q]), +send[q]) of `src`
    go to rank q, rows from rank s land at [sum(recv[:s]), +recv[s]) of `out`."""
    import torch.distributed as dist
    ns, nr = int(sum(send_rows)), int(sum(recv_rows))
    dist.all_to_all_single(out[:nr], src[:ns], output_split_sizes=[int(v) for v in recv_rows],
                           input_split_sizes=[int(v) for v in send_rows], group=group)


class _RankBuffers:
    def __init__(self, moe, R, T, d, E, k, f, fs, max_recv, device):
        import torch
        self.ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, fs), dtype=torch.uint8, device=device)
        self.layout = moe.moe_workspace_layout(T, d, E, k, f, fs)
        self.ep_ws = torch.empty(moe.moe_ep_workspace_bytes(R, E), dtype=torch.uint8, device=device)
        self.fill_base = torch.empty(E, dtype=torch.int32, device=device)
        rows = max(1, max_recv)
        self.recv = torch.empty((rows, d), dtype=torch.bfloat16, device=device)
        self.h = torch.empty((rows, f), dtype=torch.bfloat16, device=device)
        self.y_recv = torch.empty((rows, d), dtype=torch.bfloat16, device=device)
        self.h_shared = torch.empty((T, fs), dtype=torch.bfloat16, device=device) if fs else None
        self.y_shared = torch.empty((T, d), dtype=torch.bfloat16, device=device) if fs else None
        self.row_dest = torch.empty(rows, dtype=torch.int64, device=device)   # fused return: row addresses

    def view(self, moe, name, shape, dtype):
        return moe.workspace_view(self.ws, self.layout, name, shape, dtype)


class EmulatedEP:
    """R expert-parallel ranks on one device (one process, one stream)."""

    def __init__(self, R, T, d, E, k, f, f_shared=0, device="cuda", exchange="put"):
        """exchange: "put" moves rows with the library's put kernels (expert-major receive order);
        "fused" gathers x's rows straight into the receive buffers (moe_ep_dispatch_gather, no
        x_perm) and returns the results from GEMM2's own stores (moe_ep_expert_ffn_return); "a2a"
        moves them like an all-to-all-v would (source-major, device copies sized by the plans' split
        tables) and runs the source-major GEMM segments."""
        import moe_layer_router_b200 as moe
        if E % R:
            raise ValueError("E must be a multiple of R")
        if exchange not in ("put", "fused", "a2a"):
            raise ValueError("exchange must be 'put', 'fused' or 'a2a'")
        self.exchange = exchange
        self.moe, self.R, self.T, self.d, self.E, self.k, self.f, self.fs = moe, R, T, d, E, k, f, f_shared
        self.max_recv = R * T * k
        self.ranks = [_RankBuffers(moe, R, T, d, E, k, f, f_shared, self.max_recv, device) for _ in range(R)]
        import torch
        self.all_counts = torch.empty((R, E), dtype=torch.int32, device=device)

    STAGES = ["route", "permute", "dispatch", "experts", "return", "combine", "end"]

    def forward(self, xs: List, Wg, bias, W1, W3, W2, W1s, W3s, W2s, capacity_factor, cap_mode, outs: List,
                events: Optional[dict] = None) -> None:
        """xs[r]: rank r's tokens [T, d]; W1/W3/W2: all experts (rank r uses its El-expert slice);
        outs[r]: [T, d].  Capacity counts the whole batch of R * T tokens.  events: optional
        {stage: torch.cuda.Event} recorded on the current stream before each phase (STAGES)."""
        moe, R, T, d, E, k, f, fs = self.moe, self.R, self.T, self.d, self.E, self.k, self.f, self.fs
        El = E // R

        def mark(name):
            if events and events.get(name) is not None:
                events[name].record()

        C = moe.moe_capacity(R * T, E, k, capacity_factor, cap_mode)
        mark("route")
        for r, b in enumerate(self.ranks):
            moe.moe_layer_route_count(xs[r], Wg, bias, fs, T, d, E, k, f, b.ws)
        mark("permute")
        for r, b in enumerate(self.ranks):          # the all-gather of raw counts
            self.all_counts[r].copy_(b.view(moe, "counts_raw", (E,), self.all_counts.dtype))
        fused = self.exchange == "fused"
        for r, b in enumerate(self.ranks):
            moe.moe_fill_base(self.all_counts, R, r, E, b.fill_base)
            if fused:       # no x_perm: the dispatch gathers x's rows itself
                moe.moe_layer_permute_indices(xs[r], fs, T, d, E, k, f, C, b.fill_base, b.ws)
            else:
                moe.moe_layer_permute(xs[r], fs, T, d, E, k, f, C, b.fill_base, b.ws)
            moe.moe_ep_plan(self.all_counts, R, r, E, C, self.max_recv, b.ep_ws)
        recv = [b.recv for b in self.ranks]
        x_perm = [b.view(moe, "x_perm", (T * k, d), xs[r].dtype) for r, b in enumerate(self.ranks)]
        y_perm = [b.view(moe, "y_perm", (T * k, d), xs[r].dtype) for r, b in enumerate(self.ranks)]
        a2a = self.exchange == "a2a"
        if a2a:     # the plans' split sizes, on the host, as an all-to-all-v caller has them
            tabs = [moe.moe_ep_splits(b.ep_ws, R, E).cpu().tolist() for b in self.ranks]
            splits = [(t[0], t[1]) for t in tabs]
        mark("dispatch")
        if a2a:
            self._a2a([x_perm[r] for r in range(R)], recv, [sp[0] for sp in splits], [sp[1] for sp in splits])
        elif fused:
            for r, b in enumerate(self.ranks):
                moe.moe_ep_dispatch_gather(xs[r], b.view(moe, "src_token", (T * k,), self.all_counts.dtype), R, r, E,
                                           d, recv, b.ep_ws)
        else:
            for r, b in enumerate(self.ranks):
                moe.moe_ep_dispatch(x_perm[r], R, r, E, d, recv, b.ep_ws)
        mark("experts")
        for r, b in enumerate(self.ranks):
            sl = slice(r * El, (r + 1) * El)
            if fused:     # the results go straight to the tokens' ranks from GEMM2's stores
                moe.moe_ep_expert_ffn_return(b.recv, self.max_recv, R, r, E, d, f, W1[sl], W3[sl], W2[sl], b.h,
                                             xs[r], T, W1s, W3s, W2s, fs, b.h_shared, b.y_shared, y_perm, b.row_dest,
                                             b.ep_ws)
            else:
                moe.moe_ep_expert_ffn(b.recv, self.max_recv, R, r, E, d, f, W1[sl], W3[sl], W2[sl], b.h, b.y_recv,
                                      xs[r], T, W1s, W3s, W2s, fs, b.h_shared, b.y_shared, b.ep_ws, source_major=a2a)
        mark("return")
        if fused:
            pass
        elif a2a:
            self._a2a([b.y_recv for b in self.ranks], y_perm, [sp[1] for sp in splits], [sp[0] for sp in splits])
        else:
            for r, b in enumerate(self.ranks):
                moe.moe_ep_return(b.y_recv, R, r, E, d, y_perm, b.ep_ws)
        mark("combine")
        for r, b in enumerate(self.ranks):
            moe.moe_combine(y_perm[r], b.view(moe, "dest", (T, k), self.all_counts.dtype),
                            b.view(moe, "w", (T, k), _f32()), b.y_shared, T, d, k, outs[r])
        mark("end")


    @staticmethod
    def _a2a(srcs, dsts, send, recv):
        """What all_to_all_single does, on one device: rank s's rows for rank q (send[s][q], in q
        order) land in q's buffer after the rows of ranks < s (recv[q][s])."""
        R = len(srcs)
        for s in range(R):
            o = 0
            for q in range(R):
                n = int(send[s][q])
                if n:
                    at = int(sum(recv[q][:s]))
                    dsts[q][at:at + n].copy_(srcs[s][o:o + n])
                o += n


def _f32():
    import torch
    return torch.float32


def ep_layer_forward_dist(x, Wg, bias, W1_local, W3_local, W2_local, W1s, W3s, W2s, f_shared, T, d, E, k, f,
                          capacity_factor, cap_mode, out, bufs: Optional[_RankBuffers] = None, group=None):
    """One rank of an expert-parallel layer over torch.distributed (one process per GPU).
    W*_local: this rank's El experts.  The collectives: an all-gather of the raw counts and two
    all_to_all_single row exchanges; everything else runs in the library's kernels."""
    import torch
    import torch.distributed as dist
    import moe_layer_router_b200 as moe

    R, rank = dist.get_world_size(group), dist.get_rank(group)
    if bufs is None:
        bufs = _RankBuffers(moe, R, T, d, E, k, f, f_shared, R * T * k, x.device)
    C = moe.moe_capacity(R * T, E, k, capacity_factor, cap_mode)
    moe.moe_layer_route_count(x, Wg, bias, f_shared, T, d, E, k, f, bufs.ws)
    all_counts = torch.empty((R, E), dtype=torch.int32, device=x.device)
    dist.all_gather_into_tensor(all_counts, bufs.view(moe, "counts_raw", (E,), torch.int32), group=group)
    moe.moe_fill_base(all_counts, R, rank, E, bufs.fill_base)
    moe.moe_layer_permute(x, f_shared, T, d, E, k, f, C, bufs.fill_base, bufs.ws)
    moe.moe_ep_plan(all_counts, R, rank, E, C, R * T * k, bufs.ep_ws)
    send_rows, recv_rows = moe.moe_ep_splits(bufs.ep_ws, R, E).cpu().tolist()   # host split sizes
    x_perm = bufs.view(moe, "x_perm", (T * k, d), x.dtype)
    y_perm = bufs.view(moe, "y_perm", (T * k, d), x.dtype)
    exchange_rows(x_perm, send_rows, recv_rows, bufs.recv, group)
    moe.moe_ep_expert_ffn(bufs.recv, R * T * k, R, rank, E, d, f, W1_local, W3_local, W2_local, bufs.h, bufs.y_recv,
                          x, T, W1s, W3s, W2s, f_shared, bufs.h_shared, bufs.y_shared, bufs.ep_ws, source_major=True)
    exchange_rows(bufs.y_recv, recv_rows, send_rows, y_perm, group)
    moe.moe_combine(y_perm, bufs.view(moe, "dest", (T, k), torch.int32), bufs.view(moe, "w", (T, k), torch.float32),
                    bufs.y_shared, T, d, k, out)
    return bufs


class PeerBuffers:
    """Device addresses, in this process, of every rank's receive buffer and y_perm: the put
    kernels' destinations on several GPUs.  Each rank exports its two buffers (CUDA IPC handles),
    the handles are all-gathered over torch.distributed, and each rank imports the other ranks'
    (its own entry is its own pointer).  export / import_ / close default to the library's
    moe_ipc_* calls; tests pass stand-ins to check the exchange on CPU ranks."""

    def __init__(self, recv, y_perm, group=None, export=None, import_=None, close=None):
        import torch.distributed as dist
        import moe_layer_router_b200 as moe
        self._import = import_ or moe.moe_ipc_import
        self._close = close or moe.moe_ipc_close
        export = export or moe.moe_ipc_export
        self.R, self.rank = dist.get_world_size(group), dist.get_rank(group)
        mine = (export(recv), export(y_perm))
        handles = [None] * self.R
        dist.all_gather_object(handles, mine, group=group)
        self.recv, self.y_perm, self._opened = [], [], []
        for s, (h_recv, h_y) in enumerate(handles):
            if s == self.rank:
                self.recv.append(recv)
                self.y_perm.append(y_perm)
                continue
            for h, dst in ((h_recv, self.recv), (h_y, self.y_perm)):
                a = self._import(h)
                self._opened.append((a, h))
                dst.append(a)

    def close(self) -> None:
        while self._opened:
            a, h = self._opened.pop()
            self._close(a, h)


def ep_layer_forward_put_dist(x, Wg, bias, W1_local, W3_local, W2_local, W1s, W3s, W2s, f_shared, T, d, E, k, f,
                              capacity_factor, cap_mode, out, bufs: _RankBuffers, peers: PeerBuffers, group=None):
    """One rank of an expert-parallel layer whose row exchanges are peer stores into the other ranks'
    buffers (peers: PeerBuffers over bufs.recv and bufs' y_perm): a gather kernel that copies x's
    kept rows straight to their experts' ranks for the dispatch (moe_ep_dispatch_gather), GEMM2's
    own epilogue for the return (moe_ep_expert_ffn_return).  Rows arrive expert-major, so
    each local expert is one GEMM group.  The collectives: an
    all-gather of the raw counts and two barriers, each after this rank's stream has finished its
    puts, so that no rank reads a buffer before every rank has written it."""
    import torch
    import torch.distributed as dist
    import moe_layer_router_b200 as moe

    R, rank = dist.get_world_size(group), dist.get_rank(group)
    max_recv = bufs.recv.shape[0]
    C = moe.moe_capacity(R * T, E, k, capacity_factor, cap_mode)
    moe.moe_layer_route_count(x, Wg, bias, f_shared, T, d, E, k, f, bufs.ws)
    all_counts = torch.empty((R, E), dtype=torch.int32, device=x.device)
    dist.all_gather_into_tensor(all_counts, bufs.view(moe, "counts_raw", (E,), torch.int32), group=group)
    moe.moe_fill_base(all_counts, R, rank, E, bufs.fill_base)
    moe.moe_layer_permute_indices(x, f_shared, T, d, E, k, f, C, bufs.fill_base, bufs.ws)
    moe.moe_ep_plan(all_counts, R, rank, E, C, max_recv, bufs.ep_ws)
    # x's kept rows straight into the experts' ranks' receive buffers (no x_perm)
    moe.moe_ep_dispatch_gather(x, bufs.view(moe, "src_token", (T * k,), torch.int32), R, rank, E, d, peers.recv,
                               bufs.ep_ws)
    torch.cuda.current_stream(x.device).synchronize()
    dist.barrier(group=group)              # every rank's rows are in every receive buffer
    # the local experts; GEMM2 stores each result row straight into its token's rank's y_perm
    moe.moe_ep_expert_ffn_return(bufs.recv, max_recv, R, rank, E, d, f, W1_local, W3_local, W2_local, bufs.h, x, T,
                                 W1s, W3s, W2s, f_shared, bufs.h_shared, bufs.y_shared, peers.y_perm, bufs.row_dest,
                                 bufs.ep_ws)
    torch.cuda.current_stream(x.device).synchronize()
    dist.barrier(group=group)              # every result is back in its token's y_perm
    moe.moe_combine(bufs.view(moe, "y_perm", (T * k, d), x.dtype), bufs.view(moe, "dest", (T, k), torch.int32),
                    bufs.view(moe, "w", (T, k), torch.float32), bufs.y_shared, T, d, k, out)
