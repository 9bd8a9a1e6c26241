// expert_cache.cuh - expert weights in host memory, an LRU of S expert slots in HBM.
//
// [EP-DS3] section 3.2 (expert cache and preloading): experts that are not in use stay in host
// memory and the experts a batch needs are brought into HBM, evicting the least recently used
// resident expert when the slots are full.  Here the whole decision runs on the device, right
// after the batch's per-expert counts exist, so the layer needs no host round trip and stays
// capturable in a CUDA graph:
//   cache_plan_kernel   one CTA: stamps the hits, ranks the misses (ascending expert) and the
//                       free-able slots (oldest stamp first, then lower slot), pairs them rank by
//                       rank and writes the load list
//   cache_load_kernel   every SM streams the listed experts' weights (W1, W3, W2; or their fp8
//                       codes and row scales) from page-locked host memory (read directly over
//                       the host link) into their slots
// The grouped GEMMs then read weight group slot_of[e] for routed group e.  The plan also splits
// the GEMM tile prefix in two: tiles of experts that were resident before the batch (hits) and
// tiles of the experts being loaded (misses), so the hits' GEMMs can run on the layer's stream
// while the copy runs on a second stream, and only the misses' GEMMs wait for the copy
// ([EP-DS3] section 3.2: load experts asynchronously on a CUDA stream, overlapped with compute).
//
// Pairing the r-th miss with the r-th candidate slot is the same as taking misses one at a time
// and evicting the oldest candidate each time: a slot that receives a miss is stamped with the
// current batch and so leaves the candidate set, and the next-oldest candidate is next in rank.
#pragma once

#include <cstdint>

namespace moe {

// Device state (caller-owned memory, 16-byte aligned), in this order:
//   moe_cache_counters (64 B) | slot_of[E] | expert_in[S] | stamp[S] | load_expert[S] | load_slot[S]
// each int32 array padded to a multiple of 16 bytes.
struct CacheView {
    moe_cache_counters* ctr;
    int32_t* slot_of;
    int32_t* expert_in;
    int32_t* stamp;
    int32_t* load_expert;
    int32_t* load_slot;
};

inline size_t cache_pad16(size_t b) { return (b + 15) & ~size_t(15); }

inline size_t cache_layout(int E, int S, size_t off[6]) {
    size_t o = 0;
    off[0] = o; o += 64;
    off[1] = o; o += cache_pad16((size_t)E * 4);
    off[2] = o; o += cache_pad16((size_t)S * 4);
    off[3] = o; o += cache_pad16((size_t)S * 4);
    off[4] = o; o += cache_pad16((size_t)S * 4);
    off[5] = o; o += cache_pad16((size_t)S * 4);
    return o;
}

inline CacheView cache_view(void* state, int E, int S) {
    size_t off[6];
    cache_layout(E, S, off);
    char* b = static_cast<char*>(state);
    return CacheView{reinterpret_cast<moe_cache_counters*>(b + off[0]), reinterpret_cast<int32_t*>(b + off[1]),
                     reinterpret_cast<int32_t*>(b + off[2]), reinterpret_cast<int32_t*>(b + off[3]),
                     reinterpret_cast<int32_t*>(b + off[4]), reinterpret_cast<int32_t*>(b + off[5])};
}

constexpr int CACHE_MAX = 1024;   // experts and slots (one plan CTA, one thread each)

__global__ void __launch_bounds__(CACHE_MAX) cache_reset_kernel(CacheView v, int E, int S) {
    const int t = threadIdx.x;
    if (t < E) v.slot_of[t] = -1;
    if (t < S) {
        v.expert_in[t] = -1;
        v.stamp[t] = -1;
        v.load_expert[t] = -1;
        v.load_slot[t] = -1;
    }
    if (t < 8) reinterpret_cast<long long*>(v.ctr)[t] = 0;
}

// Exclusive scan over the block (blockDim.x = CACHE_MAX) of one value per thread; the total
// goes to *total.  s_warp: CACHE_MAX / 32 ints of shared memory.
__device__ __forceinline__ int cache_block_exscan(int x, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int v = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    __syncthreads();                 // s_warp free from any earlier use
    if (lane == 31) s_warp[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;            // inclusive over warps
    }
    __syncthreads();
    const int pre = (wid ? s_warp[wid - 1] : 0) + v - x;
    *total = s_warp[CACHE_MAX / 32 - 1];
    return pre;
}

// counts[e] = rows routed to expert e and kept (after capacity); an expert is needed iff > 0.
// tile_rows: rows per m-tile of the expert GEMMs; mp_hit / mp_miss [E+1]: m-tile prefixes over the
// experts that were resident before this batch / are loaded by it (the other experts count 0).
__global__ void __launch_bounds__(CACHE_MAX) cache_plan_kernel(const int32_t* __restrict__ counts, int E, int S,
                                                               CacheView v, int tile_rows, int32_t* mp_hit,
                                                               int32_t* mp_miss) {
    __shared__ int s_stamp[CACHE_MAX];
    __shared__ int s_old[CACHE_MAX];      // expert_in before this batch
    __shared__ int s_cand[CACHE_MAX];     // candidate rank -> slot
    __shared__ int s_warp[CACHE_MAX / 32];
    __shared__ int s_hits, s_cands;
    const int t = threadIdx.x;
    const int lane = t & 31, wid = t >> 5;
    const int step = (int)(v.ctr->step + 1);
    if (t == 0) { s_hits = 0; s_cands = 0; }

    // hits keep their slot and take the new stamp
    const bool need = t < E && counts[t] > 0;
    const int slot = need ? v.slot_of[t] : -1;
    const bool miss = need && slot < 0;
    if (need && slot >= 0) v.stamp[slot] = step;
    __syncthreads();
    if (need && slot >= 0) atomicAdd(&s_hits, 1);
    if (t < S) {
        s_stamp[t] = v.stamp[t];
        s_old[t] = v.expert_in[t];
    }

    // rank of each miss among the misses (ascending expert): block exclusive scan
    const unsigned bal = __ballot_sync(0xffffffffu, miss);
    if (lane == 0) s_warp[wid] = __popc(bal);
    __syncthreads();
    if (wid == 0) {
        int x = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        s_warp[lane] = x;   // inclusive
    }
    __syncthreads();
    const int n_miss = s_warp[31];
    const int miss_rank = (wid ? s_warp[wid - 1] : 0) + __popc(bal & ((1u << lane) - 1u));

    // candidate slots (not used by this batch), ranked by (stamp, slot)
    if (t < S && s_stamp[t] < step) {
        const int st = s_stamp[t];
        int r = 0;
        for (int u = 0; u < S; ++u) {
            const int su = s_stamp[u];
            r += (su < step) && (su < st || (su == st && u < t));
        }
        s_cand[r] = t;
        atomicAdd(&s_cands, 1);
    }
    __syncthreads();
    if (n_miss > s_cands) {   // the host checks S >= min(E, T*k), so this cannot happen
        if (t == 0) {
            v.ctr->loads_last = 0;
            record_error(-7 /* MOE_ERR_CHECK */);
        }
        if (t <= E) {         // no GEMM tiles in either phase
            mp_hit[t] = 0;
            mp_miss[t] = 0;
        }
        return;
    }
    // the tile prefixes of the two GEMM phases
    const int tiles = need ? (counts[t] + tile_rows - 1) / tile_rows : 0;
    int hit_total, miss_total;
    const int hit_pre = cache_block_exscan(miss ? 0 : tiles, s_warp, &hit_total);
    const int miss_pre = cache_block_exscan(miss ? tiles : 0, s_warp, &miss_total);
    if (t < E) {
        mp_hit[t] = hit_pre;
        mp_miss[t] = miss_pre;
    }
    if (t == 0) {
        mp_hit[E] = hit_total;
        mp_miss[E] = miss_total;
    }
    if (miss) {
        const int vs = s_cand[miss_rank];
        const int old = s_old[vs];
        if (old >= 0) v.slot_of[old] = -1;
        v.expert_in[vs] = t;
        v.slot_of[t] = vs;
        v.stamp[vs] = step;
        v.load_expert[miss_rank] = t;
        v.load_slot[miss_rank] = vs;
    }
    if (t == 0) {
        v.ctr->step = step;
        v.ctr->hits += s_hits;
        v.ctr->misses += n_miss;
        v.ctr->loads_last = n_miss;
    }
}

// The per-expert arrays one cache load copies: for expert e and slot v, array i moves
// per[i] 16-byte chunks from src[i] + e per[i] to dst[i] + v per[i].  bf16 experts: W1, W3, W2;
// fp8 experts: W1q, W3q, W2q and the scales s1, s3, s2.
constexpr int CACHE_MAX_ARRAYS = 6;
struct CacheCopy {
    const uint4* src[CACHE_MAX_ARRAYS];
    uint4* dst[CACHE_MAX_ARRAYS];
    long long per[CACHE_MAX_ARRAYS];
    int n;
};

// Copy the listed experts' arrays into their slots.  Every CTA takes a strided share of every
// array, so all SMs keep requests in flight.
constexpr int CACHE_LOAD_THREADS = 512;
constexpr int CACHE_LOAD_UNROLL = 8;

__global__ void __launch_bounds__(CACHE_LOAD_THREADS) cache_load_kernel(
    const moe_cache_counters* __restrict__ ctr, const int32_t* __restrict__ load_expert,
    const int32_t* __restrict__ load_slot, const CacheCopy cp) {
    const int n = (int)ctr->loads_last;
    const long long stride = (long long)gridDim.x * CACHE_LOAD_THREADS * CACHE_LOAD_UNROLL;
    for (int l = 0; l < n; ++l) {
        const long long e = load_expert[l], v = load_slot[l];
#pragma unroll 1
        for (int m = 0; m < cp.n; ++m) {
            const long long per = cp.per[m];
            const uint4* src = cp.src[m] + e * per;
            uint4* dst = cp.dst[m] + v * per;
            for (long long base = (long long)blockIdx.x * CACHE_LOAD_THREADS * CACHE_LOAD_UNROLL + threadIdx.x;
                 base < per; base += stride) {
                uint4 r[CACHE_LOAD_UNROLL];
#pragma unroll
                for (int u = 0; u < CACHE_LOAD_UNROLL; ++u) {
                    const long long i = base + (long long)u * CACHE_LOAD_THREADS;
                    if (i < per) r[u] = src[i];
                }
#pragma unroll
                for (int u = 0; u < CACHE_LOAD_UNROLL; ++u) {
                    const long long i = base + (long long)u * CACHE_LOAD_THREADS;
                    if (i < per) dst[i] = r[u];
                }
            }
        }
    }
}

}  // namespace moe
