// act_quant.cuh - fp8 e4m3 activations for the fp8 x fp8 expert GEMMs.
//
// Every activation row is quantised on its own ([EP-DS3] deployment section, w4afp8: low-bit
// weights with fp8 activations): s = amax(|x|) / 448 in fp32 (1 for an all-zero row), and each
// element becomes e4m3(fp32(x) / s), rounded to nearest even and saturating at 448 (the
// hardware conversion with .satfinite).  Two kernels apply it:
//   quant_rows_e4m3_kernel      a warp per row in two passes over the row (amax, then codes);
//                               28 registers, so many warps hide the divisions' latency
//   quant_rows_e4m3_reg_kernel  the row held in registers (read once), and optionally written
//                               to several destination rows (a token's k permuted rows)
// 16-byte loads, 8-byte stores.
#pragma once

#include <cuda_fp8.h>

namespace moe {

// rows of src (bf16, K per row; row r of the output reads src row gather[r] when gather is
// given) -> dst (e4m3, K bytes per row) and scale[r].  Rows r >= *n_rows (when n_rows is given)
// are skipped.  K % 8 == 0.
__global__ void __launch_bounds__(256) quant_rows_e4m3_kernel(const uint4* __restrict__ src,
                                                              const int32_t* __restrict__ gather,
                                                              const int32_t* __restrict__ n_rows, int rows, int K,
                                                              uint2* __restrict__ dst, float* __restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    if (n_rows && row >= __ldg(n_rows)) return;
    const long long srow = gather ? __ldg(gather + row) : row;
    const int chunks = K / 8;                     // 8 bf16 per uint4
    const uint4* s = src + srow * chunks;
    float amax = 0.f;
    for (int c = lane; c < chunks; c += 32) {
        const uint4 v = __ldg(s + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (lane == 0) scale[row] = sc;
    uint2* d = dst + (long long)row * chunks;
    for (int c = lane; c < chunks; c += 32) {
        const uint4 v = __ldg(s + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float lo = __fdiv_rn(__uint_as_float(w[i] << 16), sc);
            const float hi = __fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), sc);
            const uint32_t b0 = __nv_cvt_float_to_fp8(lo, __NV_SATFINITE, __NV_E4M3);
            const uint32_t b1 = __nv_cvt_float_to_fp8(hi, __NV_SATFINITE, __NV_E4M3);
            out[i >> 1] |= (b0 | (b1 << 8)) << (16 * (i & 1));
        }
        d[c] = make_uint2(out[0], out[1]);
    }
}

// The same recipe with each source row held in the registers of TPR threads (MAXC 16-byte
// chunks per thread, K <= 8 TPR MAXC): one HBM read of the row however long it is, all of its
// loads in flight at once.  A CTA of 256 threads takes 256 / TPR rows (TPR = 32: a warp per row,
// for short rows; 128 or 256 for long ones).  Destinations:
//   dest == nullptr: row r of src -> row r of dst / scale, rows r >= *n_rows (when given) skipped;
//   dest != nullptr: token row t -> rows dest[t k + j] (j < k, dest >= 0) of dst / scale, and,
//                    when dst_tok is given, row t of dst_tok / scale_tok (the shared expert's rows).
// Each warp store instruction writes 256 contiguous bytes of one destination row.
constexpr int QUANT_CTA = 256;

__device__ __forceinline__ float amax_bf16x8(float m, const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        m = fmaxf(m, fabsf(__uint_as_float(w[e] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
    }
    return m;
}

// 8 bf16 -> 8 e4m3 codes of e4m3(x / sc), round to nearest even, saturating
__device__ __forceinline__ uint2 e4m3x8(const uint4& v, float sc) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float lo = __fdiv_rn(__uint_as_float(w[e] << 16), sc);
        const float hi = __fdiv_rn(__uint_as_float(w[e] & 0xFFFF0000u), sc);
        const uint32_t b0 = __nv_cvt_float_to_fp8(lo, __NV_SATFINITE, __NV_E4M3);
        const uint32_t b1 = __nv_cvt_float_to_fp8(hi, __NV_SATFINITE, __NV_E4M3);
        out[e >> 1] |= (b0 | (b1 << 8)) << (16 * (e & 1));
    }
    return make_uint2(out[0], out[1]);
}

template <int TPR, int MAXC>
__global__ void __launch_bounds__(QUANT_CTA) quant_rows_e4m3_reg_kernel(
    const uint4* __restrict__ src, const int32_t* __restrict__ n_rows, long long rows, int K,
    const int32_t* __restrict__ dest, int k, uint2* __restrict__ dst, float* __restrict__ scale,
    uint2* __restrict__ dst_tok, float* __restrict__ scale_tok) {
    static_assert(TPR == 32 || TPR == 128 || TPR == 256, "a warp, or whole warps of one CTA");
    constexpr int RPC = QUANT_CTA / TPR;            // rows per CTA
    __shared__ float s_max[QUANT_CTA / 32];
    __shared__ int s_dest[RPC][32];
    const int tid = threadIdx.x % TPR, grp = threadIdx.x / TPR, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * RPC + grp;
    // rows past the end do no memory work but (TPR > 32) still meet the CTA barrier
    const bool live = row < rows && (dest || !n_rows || row < __ldg(n_rows));
    const int chunks = K / 8;
    const uint4* s = src + row * chunks;
    uint4 v[MAXC];
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
        const int c = tid + i * TPR;
        v[i] = live && c < chunks ? __ldg(s + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (dest && tid < 32) s_dest[grp][tid] = live && tid < k ? __ldg(dest + row * k + tid) : -1;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) amax = amax_bf16x8(amax, v[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (TPR > 32) {
        if (lane == 0) s_max[threadIdx.x >> 5] = amax;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < TPR / 32; ++w) amax = fmaxf(amax, s_max[grp * (TPR / 32) + w]);
    } else {
        __syncwarp();
    }
    if (!live) return;
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (!dest) {
        if (tid == 0) scale[row] = sc;
    } else {
        if (tid < k && s_dest[grp][tid] >= 0) scale[s_dest[grp][tid]] = sc;
        if (tid == 0 && dst_tok) scale_tok[row] = sc;
    }
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
        const int c = tid + i * TPR;
        if (c >= chunks) break;
        const uint2 q = e4m3x8(v[i], sc);
        if (!dest) {
            dst[row * chunks + c] = q;
        } else {
            for (int j = 0; j < k; ++j) {
                const int r = s_dest[grp][j];
                if (r >= 0) dst[(long long)r * chunks + c] = q;
            }
            if (dst_tok) dst_tok[row * chunks + c] = q;
        }
    }
}

}  // namespace moe
