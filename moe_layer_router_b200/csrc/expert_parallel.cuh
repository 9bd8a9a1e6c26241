// expert_parallel.cuh - experts split over R ranks: plan, row exchange, segment bookkeeping.
//
// [EP-KV] section 6 (the experts of a layer are spread over devices) and section 7 (two
// redistributions per layer: hidden states to the experts' ranks, outputs back to the tokens'
// ranks, then the weighted combine; all-to-all-v, point-to-point or fused kernels all qualify);
// [EP-Ops] sections 2-3 (whole experts per GPU, tokens sent to them, results returned);
// [EP-DS3] section 3.1 (_assign_experts: a uniform contiguous split).  Each rank holds E / R
// experts, rank r owning experts [r El, r El + El), El = E / R.  Both exchanges are row-range
// puts:
//   dispatch  rank r's x_perm rows for the experts of rank q are contiguous (x_perm is in global
//             expert order); they go to q's receive buffer, after the rows of ranks < r
//   return    rank q's results for the rows of rank r are contiguous in q's receive order;
//             they go back to r's y_perm at the rows they came from
// The receive buffer of rank q holds rows in (source rank, local expert) order, so the local
// grouped GEMM runs R * El row segments, segment (src, j) with the weights of local expert j.
//
// Capacity over the whole batch: the raw counts of every rank are known to every rank
// (all-gathered [R, E]); rank src keeps min(c[src][e], max(0, C - sum_{s < src} c[s][e])) rows of
// expert e, the same rows the single-batch layer keeps (token order over ranks in rank order).
#pragma once

#include <cstdint>

namespace moe {

constexpr int EP_MAX_RANKS = 64;

// Per-rank plan written by ep_plan_kernel (device memory in the EP workspace).
struct EpPlan {
    int32_t send_row0[EP_MAX_RANKS];   // first x_perm row sent to rank q
    int32_t send_rows[EP_MAX_RANKS];   // rows sent to rank q
    int32_t send_dst0[EP_MAX_RANKS];   // their first row in q's receive buffer
    int32_t back_row0[EP_MAX_RANKS];   // first receive row that came from rank s
    int32_t back_rows[EP_MAX_RANKS];   // rows that came from rank s
    int32_t back_dst0[EP_MAX_RANKS];   // their first row in s's y_perm
    int32_t recv_total;                // rows received (= rows of the local grouped GEMM)
};

// One CTA.  all_counts_raw [R, E]; C < 0: no capacity.  Writes the plan, the local segment
// offsets seg_off [R El + 1] (segment g = src * El + j) and the GEMM tile prefix mprefix
// [R El + 1] for tiles of tile_rows rows.
__global__ void __launch_bounds__(1024) ep_plan_kernel(const int32_t* __restrict__ all_counts_raw, int R, int E,
                                                       int rank, long long C, int tile_rows, EpPlan* plan,
                                                       int32_t* __restrict__ seg_off, int32_t* __restrict__ mprefix) {
    __shared__ int s_kept_sum[EP_MAX_RANKS * 2];    // [src][0]: rows src keeps for my experts
                                                    // [dst][1]: rows I keep for dst's experts
    __shared__ int s_before_me[EP_MAX_RANKS];       // rows of ranks < me kept for dst's experts
    const int El = E / R;
    const int t = threadIdx.x;
    auto kept = [&](int src, int e) -> int {
        const int c = all_counts_raw[(long long)src * E + e];
        if (C < 0) return c;
        long long before = 0;
        for (int s = 0; s < src; ++s) before += all_counts_raw[(long long)s * E + e];
        const long long room = C - before;
        return room <= 0 ? 0 : (int)(c < room ? c : room);
    };
    // per destination q: rows I keep for q's experts, and rows ranks < me keep for q's experts
    for (int q = t; q < R; q += blockDim.x) {
        int mine = 0, before = 0;
        for (int j = 0; j < El; ++j) {
            const int e = q * El + j;
            mine += kept(rank, e);
            for (int s = 0; s < rank; ++s) before += kept(s, e);
        }
        s_kept_sum[q * 2 + 1] = mine;
        s_before_me[q] = before;
    }
    // per source s: rows s keeps for my experts
    for (int s = t; s < R; s += blockDim.x) {
        int n = 0;
        for (int j = 0; j < El; ++j) n += kept(s, rank * El + j);
        s_kept_sum[s * 2] = n;
    }
    __syncthreads();
    if (t == 0) {
        int row0 = 0;
        for (int q = 0; q < R; ++q) {           // my x_perm: global expert order = rank order
            plan->send_row0[q] = row0;
            plan->send_rows[q] = s_kept_sum[q * 2 + 1];
            plan->send_dst0[q] = s_before_me[q];
            row0 += s_kept_sum[q * 2 + 1];
        }
        int r0 = 0;
        for (int s = 0; s < R; ++s) {           // my receive buffer: source-major
            plan->back_row0[s] = r0;
            plan->back_rows[s] = s_kept_sum[s * 2];
            r0 += s_kept_sum[s * 2];
        }
        plan->recv_total = r0;
    }
    // back_dst0[s]: where my experts' rows start in s's x_perm = rows s keeps for experts < rank El
    for (int s = t; s < R; s += blockDim.x) {
        int n = 0;
        for (int e = 0; e < rank * El; ++e) n += kept(s, e);
        plan->back_dst0[s] = n;
    }
    // segment offsets and tile prefix over the R El segments (one thread walks them in order)
    if (t == 0) {
        int off = 0, tiles = 0;
        for (int g = 0; g < R * El; ++g) {
            const int s = g / El, j = g % El;
            const int n = kept(s, rank * El + j);
            seg_off[g] = off;
            mprefix[g] = tiles;
            off += n;
            tiles += (n + tile_rows - 1) / tile_rows;
        }
        seg_off[R * El] = off;
        mprefix[R * El] = tiles;
    }
}

// Weight group of segment g: local expert g % El.
__global__ void ep_group_map_kernel(int R, int El, int32_t* __restrict__ group_map) {
    for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < R * El; g += gridDim.x * blockDim.x) group_map[g] = g % El;
}

struct EpDests {
    char* base[EP_MAX_RANKS];   // destination buffer of each rank (peer-mapped or local)
};

// Copy R row ranges of row_bytes each: rows [row0[q], row0[q] + rows[q]) of src go to rows
// [dst0[q], ...) of dest.base[q].  which = 0: the dispatch ranges of the plan, 1: the return ones.
// blockIdx.y = destination rank; 16-byte chunks, grid-stride over the range.
__global__ void __launch_bounds__(256) ep_put_rows_kernel(const EpPlan* __restrict__ plan, int which,
                                                          const uint4* __restrict__ src, EpDests dest,
                                                          long long row_chunks) {
    const int q = blockIdx.y;
    const int row0 = which ? plan->back_row0[q] : plan->send_row0[q];
    const int rows = which ? plan->back_rows[q] : plan->send_rows[q];
    const int dst0 = which ? plan->back_dst0[q] : plan->send_dst0[q];
    const long long n = (long long)rows * row_chunks;
    const uint4* s = src + (long long)row0 * row_chunks;
    uint4* d = reinterpret_cast<uint4*>(dest.base[q]) + (long long)dst0 * row_chunks;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        d[i] = s[i];
}

}  // namespace moe
