// grouped_gemm_w8.cuh - grouped expert GEMMs with fp8 e4m3 weights and fp32 per-row scales.
//
// The weight of output row n is e4m3(q) * s_n.  The fp8 bytes stream from HBM (half the bytes
// of bf16 weights), converter warps widen each B tile to bf16 in shared memory (exact: every
// e4m3 value is a bf16 value), the tensor cores run bf16 x bf16 -> fp32 MMAs, and the epilogue
// multiplies the accumulator of output feature n by s_n:
//   sum_i x_i * (e4m3(q_ni) * s_n) = s_n * sum_i x_i * e4m3(q_ni).
// Meant for decode, where the layer streams the expert weights once and an expert sees a few
// tokens: the weights are the MMA's M side (256 rows = two M = 128 halves) and the tokens its N
// side (N = 32 or 128), so the tensor work per k-block follows the token count, not a fixed
// 128-row tile.
//
// Roles (448 threads, one CTA per SM): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 2-5 epilogue, warps 6-13 converters.  Two rings:
//   load ring (4 stages)  A [128 x 64] bf16, 128-byte swizzle (only the first 32 rows are loaded
//                         when the tile has <= 32 rows: the other rows only feed accumulator rows
//                         that are never stored), and Q [256 x 64] fp8, unswizzled rows of 64
//                         bytes; both by TMA, so the A tile of a k-block is requested as early as
//                         its weights
//   B ring (3 stages)     [256 x 64] bf16, 128-byte swizzle, written by the converters
// Barriers: full (TMA bytes of A + Q), load_empty (MMA commit), b_full (8 converter warps),
// b_empty (MMA commit).
#pragma once

#include <cuda_fp8.h>

#include "grouped_gemm.cuh"

namespace moe {

constexpr int W8_LSTAGES = 4;     // 4 + 3 measured best of {5+2, 4+3} x {8, 12, 16} converter warps
constexpr int W8_BSTAGES = 3;
constexpr int W8_THREADS = 448;
constexpr int W8_A_BYTES = GEMM_BM * GEMM_BK * 2;   // 16 KB
constexpr int W8_Q_BYTES = 256 * GEMM_BK;           // 16 KB
constexpr int W8_B_BYTES = 256 * GEMM_BK * 2;       // 32 KB
constexpr int W8_RING_BYTES = W8_LSTAGES * (W8_A_BYTES + W8_Q_BYTES) + W8_BSTAGES * W8_B_BYTES;
constexpr int W8_SMEM_BYTES = W8_RING_BYTES + 1024 + 512;
static_assert(W8_SMEM_BYTES <= GEMM_SMEM_MAX, "w8 rings exceed shared memory");

struct W8Scales {
    const float* s0[2];   // per class: W1 scales (GEMM1) or W2 scales (GEMM2)
    const float* s1[2];   // per class: W3 scales (GEMM1), unused for GEMM2
    int group_stride[2];  // scale entries between consecutive groups (f or d; 0 for the dense class)
};

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Two e4m3 bytes (b0 at bits 0-7, b1 at bits 8-15 of `w`, selected by `sel`) -> bf16x2, exact.
// The sign goes to bf16 bit 15 and the 7 exponent/mantissa bits to bits 10..4, which reads as
// the bf16 value 2^-120 * e4m3(b) (e4m3 subnormals land on bf16 subnormals the same way); one
// bf16 multiply by 2^120 restores the value without rounding.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w, uint32_t sel) {
    uint32_t x;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(x) : "r"(w), "r"(sel));          // bytes -> high byte of each half
    x = (x & 0x80008000u) | ((x >> 4) & 0x07F007F0u);
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162 k = __floats2bfloat162_rn(0x1p120f, 0x1p120f);
    const __nv_bfloat162 r = __hmul2(v, k);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// 16 fp8 e4m3 -> 16 bf16 (two 16-byte chunks), exact.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& q, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = e4m3x2_to_bf16x2(w[i], 0x1404u);       // bytes 0, 1
        o[2 * i + 1] = e4m3x2_to_bf16x2(w[i], 0x3424u);   // bytes 2, 3
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

template <int EPI>
__global__ void __launch_bounds__(W8_THREADS, 1)
grouped_gemm_w8_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA0s,
                       const __grid_constant__ CUtensorMap tmQ0, const __grid_constant__ CUtensorMap tmQ0b,
                       const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmA1s,
                       const __grid_constant__ CUtensorMap tmQ1, const __grid_constant__ CUtensorMap tmQ1b,
                       const __grid_constant__ GemmParams p, const __grid_constant__ W8Scales sc) {
    // tmA*: A with 128-row boxes, tmA*s: 32-row boxes; tmQ*: fp8 weights (GEMM1: W1 and W3,
    // 128-row boxes; GEMM2: W2 with a 256-row box in tmQ*, tmQ*b unused)
    static_assert(EPI == EPI_SWIGLU || EPI == EPI_STORE, "expert GEMMs only");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + W8_RING_BYTES);
    uint64_t* load_empty = full_bar + W8_LSTAGES;
    uint64_t* b_full = load_empty + W8_LSTAGES;
    uint64_t* b_empty = b_full + W8_BSTAGES;
    uint64_t* tfull_bar = b_empty + W8_BSTAGES;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* drain_bar = tempty_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto sA = [&](int s) { return smem + s * W8_A_BYTES; };
    auto sQ = [&](int s) { return smem + W8_LSTAGES * W8_A_BYTES + s * W8_Q_BYTES; };
    auto sB = [&](int s) { return smem + W8_LSTAGES * (W8_A_BYTES + W8_Q_BYTES) + s * W8_B_BYTES; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < W8_LSTAGES; ++s) {
            mbar_init(full_bar + s, 1);
            mbar_init(load_empty + s, 1);
        }
        for (int s = 0; s < W8_BSTAGES; ++s) {
            mbar_init(b_full + s, 8);
            mbar_init(b_empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar + a, 1);
            mbar_init(tempty_bar + a, 128);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA0);
        prefetch_tensormap(&tmA0s);
        prefetch_tensormap(&tmQ0);
        prefetch_tensormap(&tmA1);
        prefetch_tensormap(&tmA1s);
        prefetch_tensormap(&tmQ1);
        if (EPI == EPI_SWIGLU) {
            prefetch_tensormap(&tmQ0b);
            prefetch_tensormap(&tmQ1b);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, GEMM_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    int routed_tiles;
    const int total = gemm_total_tiles(p, routed_tiles);

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_w = policy_evict_first();   // weights are read once
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const GemmClass& c = p.cls[ti.cls];
                const bool narrow = ti.rows <= 32;
                const CUtensorMap* mA = ti.cls ? (narrow ? &tmA1s : &tmA1) : (narrow ? &tmA0s : &tmA0);
                const CUtensorMap* mQ = ti.cls ? &tmQ1 : &tmQ0;
                const CUtensorMap* mQb = ti.cls ? &tmQ1b : &tmQ0b;
                const uint32_t bytes = (narrow ? 32u : 128u) * GEMM_BK * 2u + (uint32_t)W8_Q_BYTES;
                const int nk = c.K / GEMM_BK;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(load_empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(full_bar + stage, bytes);
                    tma_load_2d(sQ(stage), mQ, full_bar + stage, kb * GEMM_BK, ti.b_row, pol_w);
                    if (EPI == EPI_SWIGLU)
                        tma_load_2d(sQ(stage) + 128 * GEMM_BK, mQb, full_bar + stage, kb * GEMM_BK, ti.b_row, pol_w);
                    tma_load_2d(sA(stage), mA, full_bar + stage, kb * GEMM_BK, ti.a_row, pol_a);
                    ++issued;
                    if (++stage == W8_LSTAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {   // let the copies in flight land before the CTA exits
                const int n = issued < W8_LSTAGES ? issued : W8_LSTAGES;
                for (int i = 1; i <= n; ++i) {
                    const int q = issued - i;
                    mbar_wait(full_bar + (q % W8_LSTAGES), (uint32_t)((q / W8_LSTAGES) & 1), nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        // Swapped operands: the converted weight tile is the M side (two M = 128 halves: rows
        // 0-127 and 128-255 of the 256-row B slot), the token tile is the N side with N = 32 for
        // tiles of <= 32 rows and N = 128 otherwise.  D half h sits at columns [h N, h N + N).
        if (lane == 0) {
            int stage = 0, bstage = 0;
            uint32_t phase = 0, bphase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool any = false, ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const int nk = p.cls[ti.cls].K / GEMM_BK;
                const int nN = ti.rows <= 32 ? 32 : 128;
                const uint32_t idesc = idesc_bf16_f32(128, nN);
                if (!mbar_wait(tempty_bar + acc, acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(acc * GEMM_ACC_COLS);
                const uint32_t d1 = d0 + (uint32_t)nN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(full_bar + stage, phase, abort_flag) || !mbar_wait(b_full + bstage, bphase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t xd = smem_desc_k_sw128(sA(stage));
                    const uint64_t w0 = smem_desc_k_sw128(sB(bstage));
                    const uint64_t w1 = smem_desc_k_sw128(sB(bstage) + 128 * GEMM_BK * 2);
#pragma unroll
                    for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
                        umma_bf16(d0, w0 + 2ull * kk, xd + 2ull * kk, idesc, (kb | kk) != 0);
                        umma_bf16(d1, w1 + 2ull * kk, xd + 2ull * kk, idesc, (kb | kk) != 0);
                    }
                    umma_commit(load_empty + stage);
                    umma_commit(b_empty + bstage);
                    any = true;
                    if (++stage == W8_LSTAGES) { stage = 0; phase ^= 1u; }
                    if (++bstage == W8_BSTAGES) { bstage = 0; bphase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(tfull_bar + acc);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (any) {
                umma_commit(drain_bar);
                mbar_wait(drain_bar, 0, nullptr);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------------ converters (warps 6-13)
        // 256 rows x 4 groups of 16 fp8 per k-block; thread ct takes groups ct, ct + 256, ...
        const int ct = threadIdx.x - 6 * 32;   // 0..255
        int stage = 0, bstage = 0;
        uint32_t phase = 0, bphase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
            const int nk = p.cls[ti.cls].K / GEMM_BK;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                const bool ready = mbar_wait(full_bar + stage, phase, abort_flag) &&
                                   mbar_wait(b_empty + bstage, bphase ^ 1u, abort_flag);
                if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
                const uint8_t* q = sQ(stage);
                uint8_t* b = sB(bstage);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int u = ct + 256 * i;
                    const int row = u >> 2, grp = u & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(q + row * GEMM_BK + grp * 16);
                    uint4 lo, hi;
                    e4m3x16_to_bf16(v, lo, hi);
                    uint8_t* rb = b + (row >> 3) * 1024 + (row & 7) * 128;
                    const int c0 = (2 * grp) ^ (row & 7), c1 = (2 * grp + 1) ^ (row & 7);
                    *reinterpret_cast<uint4*>(rb + c0 * 16) = lo;
                    *reinterpret_cast<uint4*>(rb + c1 * 16) = hi;
                }
                fence_proxy_async_smem();      // generic-proxy writes -> visible to the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(b_full + bstage);
                if (++stage == W8_LSTAGES) { stage = 0; phase ^= 1u; }
                if (++bstage == W8_BSTAGES) { bstage = 0; bphase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------------ epilogue (warps 2-5)
        // TMEM lane = output feature, column = token.  Thread (sub, lane) owns feature
        // sub * 32 + lane of each 128-row half and writes it for every token of the tile: a warp
        // stores 32 consecutive features (64 bytes) of one token row per instruction.
        const int sub = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
            const GemmClass& c = p.cls[ti.cls];
            const int nN = ti.rows <= 32 ? 32 : 128;
            const bool ready = mbar_wait(tfull_bar + acc, acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t)(acc * GEMM_ACC_COLS) + ((uint32_t)(sub * 32) << 16);
            const long long row0 = c.out_row0 + ti.a_row;
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(c.out);
            const int g = ti.cls == 0 ? (ti.b_row / max(c.b_group_rows, 1)) : 0;   // expert of the tile
            const float* s0 = sc.s0[ti.cls] + (long long)g * sc.group_stride[ti.cls];
            const float* s1 = sc.s1[ti.cls] ? sc.s1[ti.cls] + (long long)g * sc.group_stride[ti.cls] : nullptr;
            if (EPI == EPI_SWIGLU) {
                const int n = ti.n_idx * 128 + sub * 32 + lane;      // gate row n of W1, up row n of W3
                const bool n_ok = n < c.n_out;
                const float sg = n_ok ? __ldg(s0 + n) : 0.f, su = n_ok ? __ldg(s1 + n) : 0.f;
#pragma unroll 1
                for (int ch = 0; ch < nN / 32; ++ch) {
                    uint32_t gv[32], uv[32];
                    __syncwarp();
                    tmem_ld_32cols(tbase + ch * 32, gv);
                    tmem_ld_32cols(tbase + nN + ch * 32, uv);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int tok = ch * 32 + j;
                        const long long orow = row0 + tok;
                        if (n_ok && tok < ti.rows && orow >= 0 && orow < c.out_rows) {
                            const float gg = __uint_as_float(gv[j]) * sg;
                            const float uu = __uint_as_float(uv[j]) * su;
                            out[orow * c.ldo + n] = __float2bfloat16_rn(gg / (1.0f + __expf(-gg)) * uu);
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    const int n = ti.n_idx * 256 + half * 128 + sub * 32 + lane;
                    const bool n_ok = n < c.n_out;
                    const float sn = n_ok ? __ldg(s0 + n) : 0.f;
#pragma unroll 1
                    for (int ch = 0; ch < nN / 32; ++ch) {
                        uint32_t v[32];
                        __syncwarp();
                        tmem_ld_32cols(tbase + half * nN + ch * 32, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int tok = ch * 32 + j;
                            const long long orow = row0 + tok;
                            if (n_ok && tok < ti.rows && orow >= 0 && orow < c.out_rows)
                                out[orow * c.ldo + n] = __float2bfloat16_rn(__uint_as_float(v[j]) * sn);
                        }
                    }
                }
            }
            __syncwarp();
            tc_fence_before();
            mbar_arrive(tempty_bar + acc);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
    }
}

}  // namespace moe
