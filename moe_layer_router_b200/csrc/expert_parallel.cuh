// expert_parallel.cuh - experts split over R ranks: plan, row exchange, segment bookkeeping.
//
// [EP-KV] section 6 (the experts of a layer are spread over devices) and section 7 (two
// redistributions per layer: hidden states to the experts' ranks, outputs back to the tokens'
// ranks, then the weighted combine; all-to-all-v, point-to-point or fused kernels all qualify);
// [EP-Ops] sections 2-3 (whole experts per GPU, tokens sent to them, results returned);
// [EP-DS3] section 3.1 (_assign_experts: a uniform contiguous split).  Each rank holds E / R
// experts, rank r owning experts [r El, r El + El), El = E / R.  Both exchanges are row-range
// puts, one range per (rank, expert):
//   dispatch  rank r's x_perm rows of expert e (contiguous: x_perm is in expert order) go to the
//             receive buffer of e's rank, which is in expert-major order: all rows of its first
//             expert (from rank 0, then rank 1, ...), then its second expert, ...
//   return    the results of rank r's rows of expert e go back to r's y_perm, at the rows they
//             had in r's x_perm
// So every local expert is one contiguous group of the local grouped GEMM and its weights are
// streamed once, however many ranks sent it rows.  (A caller that moves the rows with an
// all-to-all-v instead receives them source-major; the plan also gives that layout's segments,
// one per (source rank, local expert), which the GEMM reads through a group map.)
//
// Capacity over the whole batch: the raw counts of every rank are known to every rank
// (all-gathered [R, E]); rank src keeps min(c[src][e], max(0, C - sum_{s < src} c[s][e])) rows of
// expert e, the same rows the single-batch layer keeps (token order over ranks in rank order).
#pragma once

#include <cstdint>

namespace moe {

constexpr int EP_MAX_RANKS = 64;
constexpr int EP_MAX_EXPERTS = 1024;

// The plan of one rank, written by ep_plan_kernel into the EP workspace.
struct EpView {
    int32_t* kept;        // [R, E] rows each rank keeps per expert
    int32_t* send;        // [3, E]: src row, rows, dst row of the range of expert e (to rank e / El)
    int32_t* back;        // [3, E]: range g = s El + j: results of rank s's rows of local expert j
    int32_t* exp_off;     // [El + 1] expert-major offsets of this rank's receive buffer
    int32_t* exp_tiles;   // [El + 1] tile prefix of those groups
    int32_t* seg_off;     // [E + 1] source-major segment offsets (all-to-all-v layout)
    int32_t* seg_tiles;   // [E + 1] tile prefix of those segments
    int32_t* group_map;   // [E] segment g -> local expert g % El
    int32_t* splits;      // [2, R]: rows this rank sends to rank q, rows it receives from rank s
};

inline size_t ep_pad(size_t b) { return (b + 255) & ~size_t(255); }

inline size_t ep_layout_bytes(int R, int E, size_t off[9]) {
    const int El = E / R;
    size_t o = 0;
    off[0] = o; o += ep_pad((size_t)R * E * 4);
    off[1] = o; o += ep_pad((size_t)3 * E * 4);
    off[2] = o; o += ep_pad((size_t)3 * E * 4);
    off[3] = o; o += ep_pad((size_t)(El + 1) * 4);
    off[4] = o; o += ep_pad((size_t)(El + 1) * 4);
    off[5] = o; o += ep_pad((size_t)(E + 1) * 4);
    off[6] = o; o += ep_pad((size_t)(E + 1) * 4);
    off[7] = o; o += ep_pad((size_t)E * 4);
    off[8] = o; o += ep_pad((size_t)2 * R * 4);
    return o;
}

inline EpView ep_view(void* ws, int R, int E) {
    size_t off[9];
    ep_layout_bytes(R, E, off);
    char* b = static_cast<char*>(ws);
    auto at = [&](int i) { return reinterpret_cast<int32_t*>(b + off[i]); };
    return EpView{at(0), at(1), at(2), at(3), at(4), at(5), at(6), at(7), at(8)};
}

// Block-wide exclusive scan of one value per thread (blockDim.x = 1024); returns the prefix and
// writes the total to *total.
__device__ __forceinline__ int ep_block_exscan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;      // inclusive over warps
    }
    __syncthreads();
    const int pre = (wid ? s_warp[wid - 1] : 0) + x - v;
    *total = s_warp[31];
    __syncthreads();
    return pre;
}

// One CTA of 1024 threads (thread e = expert e).  all_counts_raw [R, E]; C < 0: no capacity.
__global__ void __launch_bounds__(1024) ep_plan_kernel(const int32_t* __restrict__ all_counts_raw, int R, int E,
                                                       int rank, long long C, int tile_rows, EpView v) {
    __shared__ int s_warp[32];
    __shared__ int s_tot_pre[EP_MAX_EXPERTS];
    const int El = E / R;
    const int e = threadIdx.x;
    // rows every rank keeps of expert e (token order over ranks), their total, mine, and below me
    int tot = 0, mine = 0, below = 0;
    if (e < E) {
        long long before = 0;
        for (int s = 0; s < R; ++s) {
            const int c = all_counts_raw[(long long)s * E + e];
            long long k = c;
            if (C >= 0) {
                const long long room = C - before;
                k = room <= 0 ? 0 : (c < room ? c : room);
            }
            v.kept[(long long)s * E + e] = (int)k;
            before += c;
            tot += (int)k;
            if (s < rank) below += (int)k;
            if (s == rank) mine = (int)k;
        }
    }
    int total_all, total_mine;
    const int tot_pre = ep_block_exscan(tot, s_warp, &total_all);      // expert-major over all ranks' buffers
    const int mine_pre = ep_block_exscan(mine, s_warp, &total_mine);   // my x_perm offsets
    if (e < E) s_tot_pre[e] = tot_pre;
    __syncthreads();    // also makes the kept[] writes above visible to the block
    if (e < E) {
        const int q = e / El;
        v.send[e] = mine_pre;                                   // my x_perm rows of expert e
        v.send[E + e] = mine;
        v.send[2 * E + e] = tot_pre - s_tot_pre[q * El] + below;   // into q's expert-major buffer
    }
    if (e < El) v.exp_off[e] = s_tot_pre[rank * El + e] - s_tot_pre[rank * El];
    if (e == 0) {
        const int last = rank * El + El - 1;
        int end = 0;
        for (int s = 0; s < R; ++s) end += v.kept[(long long)s * E + last];
        v.exp_off[El] = s_tot_pre[last] - s_tot_pre[rank * El] + end;
    }
    // return ranges: source s, local expert j -> range g = s El + j
    if (e < El) {                    // thread j: rows of each source, in source order, within expert j
        const int ge = rank * El + e;
        int acc = s_tot_pre[ge] - s_tot_pre[rank * El];
        for (int s = 0; s < R; ++s) {
            const int k = v.kept[(long long)s * E + ge];
            v.back[s * El + e] = acc;
            v.back[E + s * El + e] = k;
            acc += k;
        }
    }
    if (e < R) {                     // thread s: where my experts' rows sit in s's x_perm
        int pre = 0;
        for (int x = 0; x < rank * El; ++x) pre += v.kept[(long long)e * E + x];
        int from = 0, to = 0;
        for (int j = 0; j < El; ++j) {
            v.back[2 * E + e * El + j] = pre;
            pre += v.kept[(long long)e * E + rank * El + j];
            from += v.kept[(long long)e * E + rank * El + j];     // rank e's rows of my experts
            to += v.kept[(long long)rank * E + e * El + j];       // my rows of rank e's experts
        }
        // the split sizes of an all-to-all-v of the rows: what I send to / receive from rank e
        v.splits[e] = to;
        v.splits[R + e] = from;
    }
    __syncthreads();
    if (e == 0) {                    // tile prefixes of both layouts, and the source-major offsets
        int tiles = 0;
        for (int j = 0; j < El; ++j) {
            v.exp_tiles[j] = tiles;
            tiles += (v.exp_off[j + 1] - v.exp_off[j] + tile_rows - 1) / tile_rows;
        }
        v.exp_tiles[El] = tiles;
        int off = 0;
        tiles = 0;
        for (int g = 0; g < E; ++g) {
            const int n = v.kept[(long long)(g / El) * E + rank * El + g % El];
            v.seg_off[g] = off;
            v.seg_tiles[g] = tiles;
            off += n;
            tiles += (n + tile_rows - 1) / tile_rows;
        }
        v.seg_off[E] = off;
        v.seg_tiles[E] = tiles;
    }
    if (e < E) v.group_map[e] = e % El;
}

struct EpDests {
    char* base[EP_MAX_RANKS];   // destination buffer of each rank (peer-mapped or local)
};

// Copy the E row ranges of a plan table ([3, E]: src row, rows, dst row) of row_chunks 16-byte
// chunks per row; range r goes to dest.base[r / El].  blockIdx.y = range, grid-stride over it.
__global__ void __launch_bounds__(256) ep_put_rows_kernel(const int32_t* __restrict__ table, int E, int El,
                                                          const uint4* __restrict__ src, EpDests dest,
                                                          long long row_chunks) {
    const int r = blockIdx.y;
    const int row0 = table[r], rows = table[E + r], dst0 = table[2 * E + r];
    const long long n = (long long)rows * row_chunks;
    const uint4* s = src + (long long)row0 * row_chunks;
    uint4* d = reinterpret_cast<uint4*>(dest.base[r / El]) + (long long)dst0 * row_chunks;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        d[i] = s[i];
}

// The fused dispatch: this rank's kept rows go from x (row src_token[r] for x_perm row r) straight
// into the receive buffer of each expert's rank, so x_perm is never written or read.  Same ranges
// as the dispatch put ([3, E] send table); blockIdx.y = range, a warp per row, 16-byte chunks.
__global__ void __launch_bounds__(256) ep_gather_put_kernel(const int32_t* __restrict__ table, int E, int El,
                                                            const uint4* __restrict__ x,
                                                            const int32_t* __restrict__ src_token, EpDests dest,
                                                            int row_chunks) {
    const int r = blockIdx.y;
    const int row0 = table[r], rows = table[E + r], dst0 = table[2 * E + r];
    uint4* d = reinterpret_cast<uint4*>(dest.base[r / El]) + (long long)dst0 * row_chunks;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < rows; i += warps) {
        const uint4* src = x + (long long)__ldg(src_token + row0 + i) * row_chunks;
        uint4* dst = d + (long long)i * row_chunks;
        for (int c = lane; c < row_chunks; c += 32) dst[c] = __ldg(src + c);
    }
}

// The fused return: the byte address, in its source rank's y_perm, of every received row's
// result, from the return table ([3, E]: row in the receive buffer, rows, row in the source
// rank's y_perm; range g = s El + j goes to rank s = g / El).  GEMM2's epilogue then stores each
// result row straight there (peer stores on several GPUs), instead of a separate put kernel.
// blockIdx.y = range, grid-stride over its rows.
__global__ void __launch_bounds__(256) ep_row_dest_kernel(const int32_t* __restrict__ table, int E, int El,
                                                          EpDests dest, long long row_bytes,
                                                          long long* __restrict__ row_addr) {
    const int g = blockIdx.y;
    const int row0 = table[g], rows = table[E + g], dst0 = table[2 * E + g];
    const long long base = reinterpret_cast<long long>(dest.base[g / El]);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += gridDim.x * blockDim.x)
        row_addr[row0 + i] = base + (long long)(dst0 + i) * row_bytes;
}

}  // namespace moe
