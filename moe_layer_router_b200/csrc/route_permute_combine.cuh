// route_permute_combine.cuh - the HBM-/latency-bound stages of the layer.
//
//   topk_softmax_kernel   router top-k + renormalised softmax weights, one warp per token
//                         ([EP-DS3] §2.1 steps 1-4)
//   permute_count_kernel  per-block expert histogram + stable rank of every assignment
//   permute_scan_kernel   grid-wide scan: block bases, counts, capacity, offsets, m-tile prefix
//   permute_scatter_kernel  dest / src_token from the ranks ([EP-KV] §8, [EP-DS3] §3.1)
//   gather_rows_kernel    x_perm[dest] = x[t], one thread per 16-byte chunk
//   combine_kernel        out[t] = sum_j w * y_perm[dest] (+ y_shared), one warp per row segment
//                         ([EP-KV] §2, §7)
//   tile_prefix_kernel    m-tile prefix of the grouped GEMM from offsets (with checks)
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int PERMUTE_TOKENS = 256;   // tokens per block in the count / scatter kernels
constexpr int PERMUTE_WARPS = PERMUTE_TOKENS / 32;
constexpr int MAX_TOPK = 32;

// ---------------------------------------------------------------- block scan (<= 1024 threads)

// Exclusive scan of v over the block; returns the prefix, *total gets the block sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
    __shared__ int warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        warp_sums[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const int before = warp ? warp_sums[warp - 1] : 0;
    *total = warp_sums[nwarps - 1];
    __syncthreads();
    return before + inc - v;
}

// ---------------------------------------------------------------- router top-k

// key order: larger key first, equal keys -> lower expert index
__device__ __forceinline__ bool key_before(float ka, int ea, float kb, int eb) {
    return ka > kb || (ka == kb && ea < eb);
}

// EPL = logits held per lane (E <= 32*EPL).  One warp per token.
// With nsplit > 1 the router GEMM left nsplit partial sums (split_stride floats apart); they
// are added here in slice order 0, 1, ... and the sums are stored to logits_out.
template <int EPL>
__global__ void __launch_bounds__(256)
topk_softmax_kernel(const float* __restrict__ logits, int nsplit, long long split_stride,
                    float* __restrict__ logits_out, const float* __restrict__ bias, int T, int E, int k,
                    int32_t* __restrict__ idx, float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + (size_t)t * E;
    float L[EPL], key[EPL];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        L[i] = e < E ? __ldg(row + e) : 0.0f;
    }
    for (int sp = 1; sp < nsplit; ++sp) {      // slice order; the EPL loads of a slice go out together
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E) L[i] = __fadd_rn(L[i], __ldg(row + sp * split_stride + e));
        }
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            if (nsplit > 1 && logits_out) logits_out[(size_t)t * E + e] = L[i];
            key[i] = __fadd_rn(L[i], bias ? __ldg(bias + e) : 0.0f);   // fp32 add, no contraction
            bad |= !isfinite(key[i]) || !isfinite(L[i]);
        } else {
            L[i] = 0.0f;
            key[i] = -INFINITY;
        }
    }
    if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0) record_error(-7 /* MOE_ERR_CHECK */);
    }
    uint32_t used = 0;                 // bit i: element i of this lane already selected
    int my_e = 0;
    float my_l = -INFINITY;            // lane j < k keeps slot j
    for (int j = 0; j < k; ++j) {
        float bk = -INFINITY, bl = 0.0f;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((used >> i) & 1u) && key_before(key[i], e, bk, be)) {
                bk = key[i];
                be = e;
                bl = L[i];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (key_before(ok, oe, bk, be)) {
                bk = ok;
                be = oe;
                bl = ol;
            }
        }
        if (be < E && (be & 31) == lane) used |= 1u << (be >> 5);
        if (lane == j) {
            my_e = be < E ? be : 0;
            my_l = bl;
        }
    }
    // w_j = exp(L_j - m) / sum_sel exp(L_i - m), m = max selected logit: the softmax over
    // all E renormalised over the selected k (the common factors cancel).
    float m = lane < k ? my_l : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ex = lane < k ? expf(my_l - m) : 0.0f;
    float s = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane < k) {
        idx[(size_t)t * k + lane] = my_e;
        w[(size_t)t * k + lane] = ex / s;
    }
}

// ---------------------------------------------------------------- permutation

// Block b owns tokens [256 b, 256 b + 256).  Writes blk_cnt[b, e] (assignments to e in the
// block) and rank_local[t, j] = #{t' < t in the block : e = idx[t, j] is among idx[t', :]},
// i.e. the stable (token-order) rank of (t, j) inside its block and expert.
// Inside a warp (32 consecutive tokens) every lane sets its bit in a per-expert lane mask;
// the rank is the number of lower lanes in the mask of its expert, plus the tokens of lower
// warps routed to that expert.  Dynamic smem: (PERMUTE_WARPS * E + PERMUTE_TOKENS * k) ints.
__global__ void __launch_bounds__(PERMUTE_TOKENS)
permute_count_kernel(const int32_t* __restrict__ idx, int T, int E, int k, int32_t* __restrict__ blk_cnt,
                     int32_t* __restrict__ rank_local) {
    extern __shared__ int psm[];
    unsigned* lanes = reinterpret_cast<unsigned*>(psm);   // [PERMUTE_WARPS][E] lane masks, then warp bases
    int* sidx = psm + PERMUTE_WARPS * E;                  // [PERMUTE_TOKENS][k]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * PERMUTE_TOKENS;
    for (int i = threadIdx.x; i < PERMUTE_WARPS * E; i += blockDim.x) lanes[i] = 0u;
    for (int i = threadIdx.x; i < PERMUTE_TOKENS * k; i += blockDim.x) {
        const int t = t0 + i / k;
        int e = t < T ? __ldg(idx + (size_t)t0 * k + i) : -1;
        if (e >= E || e < -1) {
            record_error(-7 /* MOE_ERR_CHECK */);
            e = -1;
        }
        sidx[i] = e;
    }
    __syncthreads();
    const int me = warp * 32 + lane;              // token index inside the block
    const int t = t0 + me;
    unsigned* wl = lanes + warp * E;
    for (int j = 0; j < k; ++j) {
        const int e = sidx[me * k + j];
        if (e >= 0) atomicOr(wl + e, 1u << lane);
    }
    __syncthreads();
    // rank inside the warp: lower lanes whose token routes to the same expert
    const unsigned lower = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
        const int e = sidx[me * k + j];
        if (e >= 0) rank_local[(size_t)t * k + j] = __popc(wl[e] & lower);
    }
    __syncthreads();
    // per expert: exclusive prefix over warps (replaces the masks), block total
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w2 = 0; w2 < PERMUTE_WARPS; ++w2) {
            const int c = __popc(lanes[w2 * E + e]);
            lanes[w2 * E + e] = (unsigned)run;
            run += c;
        }
        blk_cnt[(size_t)blockIdx.x * E + e] = run;
    }
    __syncthreads();
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = sidx[me * k + j];
            if (e >= 0) rank_local[(size_t)t * k + j] += (int)wl[e];
        }
    }
}

// One block of 1024 threads.  In place, blk_cnt[b, e] becomes the number of assignments to
// e in blocks before b.  Then counts_raw, counts = min(raw, C - fill_base), offsets = exclusive scan
// of counts, and mprefix = exclusive scan of ceil(counts / tile_rows) (the GEMM m-tiles).
__global__ void __launch_bounds__(1024)
permute_scan_kernel(int32_t* __restrict__ blk_cnt, int nb, int E, long long C, const int32_t* __restrict__ fill_base,
                    int32_t* __restrict__ counts_raw, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ mprefix, int tile_rows) {
    __shared__ int part[1024];
    __shared__ int tot[1024];
    const int P = blockDim.x / E;                 // partitions of the block range per expert
    const int tid = threadIdx.x;
    const int e = tid % E, pi = tid / E;
    const bool active = pi < P;
    const int chunk = (nb + P - 1) / P;
    const int b0 = pi * chunk, b1 = min(nb, b0 + chunk);
    int s = 0;
    if (active)
        for (int b = b0; b < b1; ++b) s += blk_cnt[(size_t)b * E + e];
    part[tid] = s;
    __syncthreads();
    if (active && pi == 0) {
        int run = 0;
        for (int q = 0; q < P; ++q) {
            const int v = part[q * E + e];
            part[q * E + e] = run;
            run += v;
        }
        tot[e] = run;
    }
    __syncthreads();
    if (active) {
        int run = part[tid];
        for (int b = b0; b < b1; ++b) {
            const int c = blk_cnt[(size_t)b * E + e];
            blk_cnt[(size_t)b * E + e] = run;
            run += c;
        }
    }
    // kept: the first C - fill_base[e] assignments in token order (fill_base: assignments of
    // the same expert from tokens before this batch, on other ranks; 0 without sharding)
    const int raw = tid < E ? tot[tid] : 0;
    const long long room = tid < E ? C - (fill_base ? (long long)fill_base[tid] : 0ll) : 0;
    const int kept = tid < E ? (C < 0 ? raw : (int)max(0ll, min((long long)raw, room))) : 0;
    int total;
    const int off = block_exclusive_scan(kept, &total);
    const int mt = (kept + tile_rows - 1) / tile_rows;
    int mtotal;
    const int moff = block_exclusive_scan(mt, &mtotal);
    if (tid < E) {
        counts_raw[tid] = raw;
        counts[tid] = kept;
        offsets[tid] = off;
        mprefix[tid] = moff;
    }
    if (tid == 0) {
        offsets[E] = total;
        mprefix[E] = mtotal;
    }
}

__global__ void __launch_bounds__(PERMUTE_TOKENS)
permute_scatter_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ rank_local,
                       const int32_t* __restrict__ blk_base, const int32_t* __restrict__ offsets, int T, int E,
                       int k, long long C, const int32_t* __restrict__ fill_base, int32_t* __restrict__ dest,
                       int32_t* __restrict__ src_token) {
    const int t = blockIdx.x * PERMUTE_TOKENS + threadIdx.x;
    if (t >= T) return;
    for (int j = 0; j < k; ++j) {
        const int e = __ldg(idx + (size_t)t * k + j);
        int d = -1;
        if (e >= 0 && e < E) {
            const long long r = (long long)__ldg(blk_base + (size_t)blockIdx.x * E + e) + __ldg(rank_local + (size_t)t * k + j);
            const long long base = fill_base ? (long long)__ldg(fill_base + e) : 0ll;
            if (C < 0 || base + r < C) {
                d = __ldg(offsets + e) + (int)r;
                src_token[d] = t;
            }
        }
        dest[(size_t)t * k + j] = d;
    }
}

// x_perm[dest[t, j]] = x[t].  One thread per 16-byte chunk of a token row: it reads the
// chunk once and writes it to each kept destination (T*d/8 threads, so small batches still
// spread over every SM).
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ dest, int T, int d, int k,
                   uint4* __restrict__ x_perm) {
    const int nvec = d / 8;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)T * nvec) return;
    const int t = (int)(i / nvec), c = (int)(i - (long long)t * nvec);
    const uint4 v = __ldg(x + i);
    const int32_t* dt = dest + (size_t)t * k;
    for (int j = 0; j < k; ++j) {
        const int r = __ldg(dt + j);
        if (r >= 0) x_perm[(size_t)r * nvec + c] = v;
    }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// out[t] = bf16( sum_{j=0..k-1, dest>=0} w[t,j] * y_perm[dest[t,j]] + y_shared[t] ), fp32 FMA in
// j order.  One warp per (token, segment of 32*seg_chunks 16-byte chunks): lane j < k loads
// slot j's row and weight once and shuffles them; loads of four slots are in flight at a
// time.  seg_chunks is chosen on the host so that small batches still fill the GPU.
__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ dest, const float* __restrict__ w,
               const uint4* __restrict__ y_shared, int T, int d, int k, int seg_chunks, uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int nvec = d / 8;
    const int seg_len = 32 * seg_chunks;
    const int nseg = (nvec + seg_len - 1) / seg_len;
    const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= (long long)T * nseg) return;
    const int t = (int)(wid / nseg), sg = (int)(wid - (long long)t * nseg);
    const int dj = lane < k ? __ldg(dest + (size_t)t * k + lane) : -1;
    const float wj = lane < k ? __ldg(w + (size_t)t * k + lane) : 0.0f;
    const int c_end = min(nvec, (sg + 1) * seg_len);
    for (int c = sg * seg_len + lane; c - lane < c_end; c += 32) {
        const bool ok = c < c_end;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        for (int j = 0; j < k; j += 4) {
            int r[4];
            float wv[4];
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                r[q] = __shfl_sync(0xffffffffu, dj, (j + q) & 31);
                wv[q] = __shfl_sync(0xffffffffu, wj, (j + q) & 31);
                if (j + q >= k) r[q] = -1;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                v[q] = (ok && r[q] >= 0) ? __ldg(y_perm + (size_t)r[q] * nvec + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (r[q] >= 0) {
                    float f[8];
                    bf16x8_to_f32(v[q], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = fmaf(wv[q], f[e], acc[e]);
                }
            }
        }
        if (ok) {
            if (y_shared) {
                float f[8];
                bf16x8_to_f32(__ldg(y_shared + (size_t)t * nvec + c), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], f[e]);
            }
            out[(size_t)t * nvec + c] = make_uint4(f32x2_to_bf16x2(acc[0], acc[1]), f32x2_to_bf16x2(acc[2], acc[3]),
                                                   f32x2_to_bf16x2(acc[4], acc[5]), f32x2_to_bf16x2(acc[6], acc[7]));
        }
    }
}

// fill_base[e] = sum over ranks g < rank of all_counts[g, e]: the assignments to expert e
// from the token batches before this rank's in global token order.
__global__ void fill_base_kernel(const int32_t* __restrict__ all_counts, int G, int rank, int E,
                                 int32_t* __restrict__ fill_base) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    long long s = 0;
    for (int g = 0; g < rank && g < G; ++g) s += all_counts[(size_t)g * E + e];
    fill_base[e] = (int32_t)min(s, (long long)0x7fffffff);
}

// Selection bias from the overflow of the last batch ([EP-DS3] §2.1 expert_bias update):
// bias_e = -clamp((counts_raw_e - C) / C, -1, 1) in fp32, IEEE division (C > 0).
__global__ void update_bias_kernel(const int32_t* __restrict__ counts_raw, int E, long long C,
                                   float* __restrict__ bias) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const float over = (float)((long long)counts_raw[e] - C);
    const float r = fminf(fmaxf(__fdiv_rn(over, (float)C), -1.0f), 1.0f);
    bias[e] = -r;
}

// mprefix = exclusive scan of ceil((offsets[e+1]-offsets[e]) / tile_rows).  If offsets are not a
// monotone sequence starting at 0 and ending <= max_rows, records MOE_ERR_CHECK and
// writes an all-zero prefix (no GEMM tile runs).
__global__ void __launch_bounds__(1024)
tile_prefix_kernel(const int32_t* __restrict__ offsets, int E, int max_rows, int tile_rows,
                   int32_t* __restrict__ mprefix) {
    __shared__ int bad;
    const int e = threadIdx.x;
    if (e == 0) bad = 0;
    __syncthreads();
    int mt = 0;
    if (e < E) {
        const int a = offsets[e], b = offsets[e + 1];
        if (a < 0 || b < a || b > max_rows || (e == 0 && a != 0)) bad = 1;
        mt = (b - a + tile_rows - 1) / tile_rows;
    }
    __syncthreads();
    if (bad) mt = 0;
    int total;
    const int moff = block_exclusive_scan(mt, &total);
    if (e < E) mprefix[e] = moff;
    if (e == 0) {
        mprefix[E] = total;
        if (bad) record_error(-7 /* MOE_ERR_CHECK */);
    }
}

}  // namespace moe
