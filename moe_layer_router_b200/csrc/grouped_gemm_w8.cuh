// grouped_gemm_w8.cuh - grouped expert GEMMs with fp8 e4m3 weights and fp32 per-row scales.
//
// The weight of output row n is e4m3(q) * s_n.  The fp8 bytes stream from HBM (half the bytes
// of bf16 weights), converter warps widen each weight tile to bf16 (exact: every e4m3 value is a
// bf16 value), the tensor cores run bf16 x bf16 -> fp32 MMAs, and the epilogue multiplies the
// accumulator of output feature n by s_n:
//   sum_i x_i * (e4m3(q_ni) * s_n) = s_n * sum_i x_i * e4m3(q_ni).
// Meant for decode, where the layer streams the expert weights once and an expert sees a few
// tokens: the weights are the MMA's M side (256 rows = two M = 128 halves) and the tokens its N
// side (N = 32 for tiles of <= 32 rows, else 128), so the tensor work per k-block follows the
// token count.  The converted weights never touch shared memory: the converters store them into
// tensor memory with tcgen05.st and the MMAs read their A operand from there.
//
// Roles (480 threads, one CTA per SM): warp 0 loads the fp8 weights, warp 14 loads the token
// rows, warp 1 allocates TMEM and issues the MMAs, warps 2-5 run the epilogue, warps 6-13 convert
// (warp w owns TMEM lanes 32 (w % 4) .. +31 of weight half (w - 6) / 4, one weight row per thread).
//   fp8 ring (8 stages)     Q [256 x 64] fp8, 64-byte rows with 64-byte swizzle (conflict-free row
//                           reads); a slot is free again as soon as the converters have read it,
//                           so up to 128 KB of weights per SM stay in flight
//   token ring (4 stages)   A [128 x 64] bf16 token rows, 128-byte swizzle (only the first 32 rows
//                           when the tile has <= 32 rows: the other rows only feed accumulator
//                           columns that are never stored); freed by the MMA commit
//   TMEM columns            [0, 192): 3 stages of converted weights, 64 columns each (half h at
//                           +32 h, two bf16 per column); [192, 320) and [320, 448): two accumulator
//                           slots of 128 columns; a tile of <= 32 rows takes one slot (2 x 32
//                           columns), a wider tile both (2 x 128 columns)
// Barriers: q_full / a_full (TMA bytes), q_empty / w_full (8 converter warps), a_empty / w_empty
// (MMA commit), acc_full / acc_empty per slot.
#pragma once

#include <cuda_fp8.h>

#include "grouped_gemm.cuh"

namespace moe {

constexpr int W8_QSTAGES = 8;
constexpr int W8_ASTAGES = 4;
constexpr int W8_TSTAGES = 3;
constexpr int W8_CONV_WARPS = 8;
constexpr int W8_THREADS = (7 + W8_CONV_WARPS) * 32;
constexpr int W8_A_BYTES = GEMM_BM * GEMM_BK * 2;   // 16 KB
constexpr int W8_Q_BYTES = 256 * GEMM_BK;           // 16 KB
constexpr int W8_RING_BYTES = W8_QSTAGES * W8_Q_BYTES + W8_ASTAGES * W8_A_BYTES;
constexpr int W8_SMEM_BYTES = W8_RING_BYTES + 1024 + 512;
constexpr uint32_t W8_TCOL_W = 0;                    // converted weights
constexpr uint32_t W8_TCOL_ACC = 64 * W8_TSTAGES;    // accumulator slots
static_assert(W8_SMEM_BYTES <= GEMM_SMEM_MAX, "w8 ring exceeds shared memory");
static_assert(W8_TCOL_ACC + 256 <= GEMM_TMEM_COLS, "w8 TMEM columns");

// 32 lanes x 32 columns of 32-bit into TMEM: thread i writes v[0..31] to lane (taddr.lane + i),
// columns taddr.col .. +31; the address is the same for the whole warp.
__device__ __forceinline__ void tmem_st_32cols(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]),
        "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulate; one thread issues.  A (M x 16,
// K-major) sits in lanes 0..M-1, two bf16 per 32-bit column (even K in the low half), 8 columns.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct W8Scales {
    const float* s0[2];   // per class: W1 scales (GEMM1) or W2 scales (GEMM2)
    const float* s1[2];   // per class: W3 scales (GEMM1), unused for GEMM2
    int group_stride[2];  // scale entries between consecutive groups (f or d; 0 for the dense class)
};

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

// 16 fp8 e4m3 -> 16 bf16 as 8 packed words (element 2j in the low half of word j), exact.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& q, uint32_t* o) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = e4m3x2_to_bf16x2(w[i], 0x1404u);       // bytes 0, 1
        o[2 * i + 1] = e4m3x2_to_bf16x2(w[i], 0x3424u);   // bytes 2, 3
    }
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
    uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + W8_RING_BYTES);
    uint64_t* q_empty = q_full + W8_QSTAGES;
    uint64_t* a_full = q_empty + W8_QSTAGES;
    uint64_t* a_empty = a_full + W8_ASTAGES;
    uint64_t* w_full = a_empty + W8_ASTAGES;
    uint64_t* w_empty = w_full + W8_TSTAGES;
    uint64_t* acc_full = w_empty + W8_TSTAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain_bar = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto sQ = [&](int s) { return smem + s * W8_Q_BYTES; };
    auto sA = [&](int s) { return smem + W8_QSTAGES * W8_Q_BYTES + s * W8_A_BYTES; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < W8_QSTAGES; ++s) {
            mbar_init(q_full + s, 1);
            mbar_init(q_empty + s, W8_CONV_WARPS);
        }
        for (int s = 0; s < W8_ASTAGES; ++s) {
            mbar_init(a_full + s, 1);
            mbar_init(a_empty + s, 1);
        }
        for (int s = 0; s < W8_TSTAGES; ++s) {
            mbar_init(w_full + s, W8_CONV_WARPS);
            mbar_init(w_empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full + a, 1);
            mbar_init(acc_empty + a, 4);       // one arrival per epilogue warp
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ0);
        prefetch_tensormap(&tmQ1);
        if (EPI == EPI_SWIGLU) {
            prefetch_tensormap(&tmQ0b);
            prefetch_tensormap(&tmQ1b);
        }
    }
    if (warp == 14 && lane == 0) {
        prefetch_tensormap(&tmA0);
        prefetch_tensormap(&tmA0s);
        prefetch_tensormap(&tmA1);
        prefetch_tensormap(&tmA1s);
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
        // ------------------------------------------------------------------ fp8 weight producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();   // weights are read once
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const GemmClass& c = p.cls[ti.cls];
                const CUtensorMap* mQ = ti.cls ? &tmQ1 : &tmQ0;
                const CUtensorMap* mQb = ti.cls ? &tmQ1b : &tmQ0b;
                const int nk = c.K / GEMM_BK;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(q_empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(q_full + stage, (uint32_t)W8_Q_BYTES);
                    tma_load_2d(sQ(stage), mQ, q_full + stage, kb * GEMM_BK, ti.b_row, pol_w);
                    if (EPI == EPI_SWIGLU)
                        tma_load_2d(sQ(stage) + 128 * GEMM_BK, mQb, q_full + stage, kb * GEMM_BK, ti.b_row, pol_w);
                    ++issued;
                    if (++stage == W8_QSTAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {   // let the copies in flight land before the CTA exits
                const int n = issued < W8_QSTAGES ? issued : W8_QSTAGES;
                for (int i = 1; i <= n; ++i) {
                    const int q = issued - i;
                    mbar_wait(q_full + (q % W8_QSTAGES), (uint32_t)((q / W8_QSTAGES) & 1), nullptr);
                }
            }
        }
    } else if (warp == 14) {
        // ------------------------------------------------------------------ token-row producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const GemmClass& c = p.cls[ti.cls];
                const bool narrow = ti.rows <= 32;
                const CUtensorMap* mA = ti.cls ? (narrow ? &tmA1s : &tmA1) : (narrow ? &tmA0s : &tmA0);
                const uint32_t bytes = (narrow ? 32u : 128u) * GEMM_BK * 2u;
                const int nk = c.K / GEMM_BK;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(a_empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(a_full + stage, bytes);
                    tma_load_2d(sA(stage), mA, a_full + stage, kb * GEMM_BK, ti.a_row, pol_a);
                    ++issued;
                    if (++stage == W8_ASTAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                const int n = issued < W8_ASTAGES ? issued : W8_ASTAGES;
                for (int i = 1; i <= n; ++i) {
                    const int q = issued - i;
                    mbar_wait(a_full + (q % W8_ASTAGES), (uint32_t)((q / W8_ASTAGES) & 1), nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        // D half h (weight rows 128 h .. 128 h + 127) of a tile with N token columns sits at
        // columns [h N, h N + N) of its accumulator region.
        if (lane == 0) {
            int stage = 0, wstage = 0, slot = 0;
            uint32_t phase = 0, wphase = 0;
            uint32_t aph[2] = {0, 0};
            bool any = false, ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const int nk = p.cls[ti.cls].K / GEMM_BK;
                const bool wide = ti.rows > 32;
                const int nN = wide ? 128 : 32;
                const uint32_t idesc = idesc_bf16_f32(128, nN);
                if (wide) {
                    if (!mbar_wait(acc_empty + 0, aph[0] ^ 1u, abort_flag) ||
                        !mbar_wait(acc_empty + 1, aph[1] ^ 1u, abort_flag))
                        break;
                } else if (!mbar_wait(acc_empty + slot, aph[slot] ^ 1u, abort_flag)) {
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + W8_TCOL_ACC + (wide ? 0u : 128u * (uint32_t)slot);
                const uint32_t d1 = d0 + (uint32_t)nN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(a_full + stage, phase, abort_flag) || !mbar_wait(w_full + wstage, wphase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t xd = smem_desc_k_sw128(sA(stage));
                    const uint32_t w0 = tmem_base + W8_TCOL_W + 64u * (uint32_t)wstage;
#pragma unroll
                    for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
                        umma_bf16_ts(d0, w0 + 8u * kk, xd + 2ull * kk, idesc, (kb | kk) != 0);
                        umma_bf16_ts(d1, w0 + 32u + 8u * kk, xd + 2ull * kk, idesc, (kb | kk) != 0);
                    }
                    umma_commit(a_empty + stage);
                    umma_commit(w_empty + wstage);
                    any = true;
                    if (++stage == W8_ASTAGES) { stage = 0; phase ^= 1u; }
                    if (++wstage == W8_TSTAGES) { wstage = 0; wphase ^= 1u; }
                }
                if (!ok) break;
                if (wide) {
                    umma_commit(acc_full + 0);
                    umma_commit(acc_full + 1);
                    aph[0] ^= 1u;
                    aph[1] ^= 1u;
                } else {
                    umma_commit(acc_full + slot);
                    aph[slot] ^= 1u;
                    slot ^= 1;
                }
            }
            if (any) {
                umma_commit(drain_bar);
                mbar_wait(drain_bar, 0, nullptr);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------------ converters (warps 6-13)
        // Thread (warp w, lane i) converts weight row r = 128 h + 32 (w % 4) + i, h = (w - 6) / 4:
        // 64 fp8 bytes, chunk g of the row stored at chunk g ^ ((r >> 1) & 3) (64-byte swizzle, so
        // eight consecutive rows read eight different bank groups), into 32 TMEM columns of lane
        // 32 (w % 4) + i, weight half h of the stage.
        const int half = (warp - 6) >> 2;
        const int quarter = warp & 3;
        const int r = half * 128 + quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int stage = 0, wstage = 0;
        uint32_t phase = 0, wphase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
            const int nk = p.cls[ti.cls].K / GEMM_BK;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                const bool ready = mbar_wait(q_full + stage, phase, abort_flag) &&
                                   mbar_wait(w_empty + wstage, wphase ^ 1u, abort_flag);
                if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
                tc_fence_after();
                const uint8_t* q = sQ(stage) + r * GEMM_BK;
                uint4 v[4];
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    v[g] = *reinterpret_cast<const uint4*>(q + ((g ^ ((r >> 1) & 3)) << 4));
                uint32_t o[32];
#pragma unroll
                for (int g = 0; g < 4; ++g) e4m3x16_to_bf16(v[g], o + 8 * g);
                __syncwarp();
                if (lane == 0) mbar_arrive(q_empty + stage);     // the fp8 slot has been read
                tmem_st_32cols(tmem_base + lane_addr + W8_TCOL_W + 64u * (uint32_t)wstage + 32u * (uint32_t)half, o);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(w_full + wstage);
                if (++stage == W8_QSTAGES) { stage = 0; phase ^= 1u; }
                if (++wstage == W8_TSTAGES) { wstage = 0; wphase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------------ epilogue (warps 2-5)
        // TMEM lane = output feature, column = token.  Thread (sub, lane) owns feature
        // sub * 32 + lane of each 128-row half and writes it for every token of the tile: a warp
        // stores 32 consecutive features (64 bytes) of one token row per instruction.
        const int sub = warp & 3;
        int slot = 0;
        uint32_t aph[2] = {0, 0};
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
            const GemmClass& c = p.cls[ti.cls];
            const bool wide = ti.rows > 32;
            const int nN = wide ? 128 : 32;
            bool ready;
            if (wide)
                ready = mbar_wait(acc_full + 0, aph[0], abort_flag) && mbar_wait(acc_full + 1, aph[1], abort_flag);
            else
                ready = mbar_wait(acc_full + slot, aph[slot], abort_flag);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + W8_TCOL_ACC + (wide ? 0u : 128u * (uint32_t)slot) +
                                   ((uint32_t)(sub * 32) << 16);
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
                            out[orow * c.ldo + n] = __float2bfloat16_rn(swiglu_f32(gg, uu));
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const int n = ti.n_idx * 256 + hh * 128 + sub * 32 + lane;
                    const bool n_ok = n < c.n_out;
                    const float sn = n_ok ? __ldg(s0 + n) : 0.f;
#pragma unroll 1
                    for (int ch = 0; ch < nN / 32; ++ch) {
                        uint32_t v[32];
                        __syncwarp();
                        tmem_ld_32cols(tbase + hh * nN + ch * 32, v);
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
            tc_fence_before();
            __syncwarp();                     // every lane's tensor-memory reads are done
            if (wide) {
                if (lane == 0) {
                    mbar_arrive_relaxed(acc_empty + 0);
                    mbar_arrive_relaxed(acc_empty + 1);
                }
                aph[0] ^= 1u;
                aph[1] ^= 1u;
            } else {
                if (lane == 0) mbar_arrive_relaxed(acc_empty + slot);
                aph[slot] ^= 1u;
                slot ^= 1;
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
    }
}

}  // namespace moe
