// grouped_gemm.cuh - persistent tcgen05 grouped GEMM for the router and the expert FFN.
//
// One kernel template serves three products, all of the form  D = A * B^T  with A and B
// K-major bf16 and D accumulated in fp32 in tensor memory (TMEM):
//   EPI_LOGITS : router,  A = x [T,d],           B = Wg [E,d]         -> fp32 logits [T,E]
//   EPI_SWIGLU : GEMM1,   A = x_perm rows of e,  B = W1_e|W3_e tiles  -> h = bf16(silu(g)*u)
//   EPI_STORE  : GEMM2,   A = h rows of e,       B = W2_e             -> bf16 y
// (the SwiGLU expert of [EP-KV] §1, grouped per expert as in [EP-KV] §8).
//
// Work decomposition.  Output tiles are BM=128 rows x BN columns.  A "class" is a set of
// groups sharing tensor maps: class 0 = the routed experts (group g owns rows
// [offsets[g], offsets[g+1]) of A, read from device memory), class 1 = one dense group
// (all rows of its own A; the router, or the always-on shared expert).  The per-group
// m-tile counts are prefix-summed on the device (mprefix), so no host synchronisation is
// needed: every CTA of the persistent grid walks tiles t = blockIdx.x, +gridDim.x, ...
// Inside a group the m index runs fastest, so CTAs working at the same time share one
// weight tile (read once from HBM, then from L2) and the group's A rows stay in L2.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile [128 x 64] + B tile [BN x 64] per k-block into a
//               4-stage ring of 128-byte-swizzled shared memory.
//   warp 1      TMEM allocator + MMA issuer: 4 x tcgen05.mma (M=128, N=BN, K=16) per
//               k-block into one of two TMEM accumulators (2 x 256 columns).
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, SwiGLU / bf16 / fp32 conversion,
//               masked 16-byte stores.  Warp w reads TMEM lanes 32*(w%4) .. +31, i.e.
//               output rows 32*(w%4) + lane of the tile.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;                       // one 128-byte swizzle row of bf16
constexpr int GEMM_STAGES = 4;                        // stages when B tiles are 256 rows
constexpr int GEMM_MAX_STAGES = 12;
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;   // 16 KB
constexpr int GEMM_B_BYTES = 256 * GEMM_BK * 2;       // 32 KB (N <= 256)
constexpr int GEMM_ACC_COLS = 256;
constexpr int GEMM_TMEM_COLS = 512;
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_SMEM_MAX = 232448;                 // 227 KB opt-in per CTA
constexpr int GEMM_SMEM_BYTES = GEMM_STAGES * (GEMM_A_BYTES + GEMM_B_BYTES) + 1024 + 256;

// Shared memory of a ring of `stages` slots, each one A tile and one B slot of b_slot bytes.
__host__ __device__ constexpr int gemm_smem_bytes(int stages, int b_slot) {
    return stages * (GEMM_A_BYTES + b_slot) + 1024 + 256;
}

enum { EPI_LOGITS = 0, EPI_SWIGLU = 1, EPI_STORE = 2 };

struct GemmClass {
    int K;              // reduction length per tile (per split), multiple of 64
    int n_out;          // valid output columns
    int ntiles;         // tiles along N
    int b_group_rows;   // rows between consecutive groups in the B tensor(s)
    int b_tile_rows;    // B rows loaded per tile per map (128 SwiGLU half, 256 store, padded E router)
    int mma_n;          // MMA N
    void* out;          // output base pointer
    long long ldo;      // output row stride in elements
    long long out_row0; // added to the tile's A row to get the output row
    long long out_rows; // output rows available (stores at or beyond are dropped)
    int ksplit;         // dense class: K is cut into ksplit slices of K each (>= 1)
    long long split_stride;  // output elements between the partial results of two slices
    // fp8 operands (F8 kernels): the fp32 accumulator of A row r, output column n of weight
    // group g is multiplied by a_scale[r] * b_scale[g * b_scale_stride + n] (b_scale2: the up
    // projection of a SwiGLU tile)
    const float* a_scale;
    const float* b_scale;
    const float* b_scale2;
    long long b_scale_stride;
    // nullable: output row r (A-row index) goes to the byte address row_addr[r] instead of
    // out + (out_row0 + r) * ldo (rows of another rank's buffer, for the fused return exchange)
    const long long* row_addr;
};

struct GemmParams {
    GemmClass cls[2];
    const int32_t* offsets;  // [E+1] routed row offsets (class 0), nullptr = no class 0
    const int32_t* mprefix;  // [E+1] prefix of per-group m-tile counts (class 0)
    int E;
    int dense_rows;          // rows of class 1 (0 = no class 1)
    int stages;              // ring slots (<= GEMM_MAX_STAGES)
    int b_slot;              // bytes of one B slot (multiple of 1024)
    const int32_t* group_map;  // [E] routed group -> weight group (expert cache slots); nullptr = identity
    int swap_max;              // pair kernel: tail tiles of at most this many rows run swapped (0 = none)
};

// Weight group that routed group g reads its B rows from.
__device__ __forceinline__ int gemm_weight_group(const GemmParams& p, int g) {
    return p.group_map ? __ldg(p.group_map + g) : g;
}

struct TileInfo {
    int cls;
    int a_row;   // first A row of the tile
    int rows;    // valid rows (<= 128)
    int b_row;   // first B row (gate half for SwiGLU)
    int n_idx;   // tile index along N
    int ks;      // K slice (dense class with ksplit > 1)
};

__device__ __forceinline__ int gemm_total_tiles(const GemmParams& p, int& routed_tiles) {
    routed_tiles = p.offsets ? __ldg(p.mprefix + p.E) * p.cls[0].ntiles : 0;
    const int dense =
        p.dense_rows ? ((p.dense_rows + GEMM_BM - 1) / GEMM_BM) * p.cls[1].ntiles * p.cls[1].ksplit : 0;
    return routed_tiles + dense;
}

__device__ __forceinline__ TileInfo gemm_decode_tile(const GemmParams& p, int t, int routed_tiles) {
    TileInfo ti;
    if (t < routed_tiles) {
        const GemmClass& c = p.cls[0];
        const int q = t / c.ntiles;              // virtual m-tile index
        int lo = 0, hi = p.E;                    // mprefix[lo] <= q < mprefix[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(p.mprefix + mid) <= q) lo = mid; else hi = mid;
        }
        const int g = lo;
        const int mp = __ldg(p.mprefix + g);
        const int mt = __ldg(p.mprefix + g + 1) - mp;
        const int local = t - mp * c.ntiles;
        const int m = local % mt, n = local / mt;
        const int r0 = __ldg(p.offsets + g) + m * GEMM_BM;
        ti.cls = 0;
        ti.a_row = r0;
        ti.rows = min(GEMM_BM, __ldg(p.offsets + g + 1) - r0);
        ti.n_idx = n;
        ti.b_row = gemm_weight_group(p, g) * c.b_group_rows + n * c.b_tile_rows;
        ti.ks = 0;
    } else {
        const GemmClass& c = p.cls[1];
        const int mt = (p.dense_rows + GEMM_BM - 1) / GEMM_BM;
        const int local = t - routed_tiles;
        const int m = local % mt, rest = local / mt;
        const int n = rest % c.ntiles;
        ti.cls = 1;
        ti.a_row = m * GEMM_BM;
        ti.rows = min(GEMM_BM, p.dense_rows - ti.a_row);
        ti.n_idx = n;
        ti.b_row = n * c.b_tile_rows;
        ti.ks = rest / c.ntiles;
    }
    return ti;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// SwiGLU of one gate/up accumulator pair: silu(g) u with silu(g) = g / (1 + e^-g).  The fast
// divide (two ulp) is ample for a value rounded to bf16 next; for g below about -87 the
// denominator overflows and the result is the correct limit 0.
__device__ __forceinline__ float swiglu_f32(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// fp8 products: 32 accumulator columns times the A row's scale sa and the columns' weight
// scales sb[0..32) (16-byte aligned; fp8 outputs come in whole 128-column tiles).
__device__ __forceinline__ void scale_cols32(uint32_t (&v)[32], float sa, const float* sb) {
    const float4* s4 = reinterpret_cast<const float4*>(sb);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 c = __ldg(s4 + q);
        v[4 * q + 0] = __float_as_uint(__uint_as_float(v[4 * q + 0]) * sa * c.x);
        v[4 * q + 1] = __float_as_uint(__uint_as_float(v[4 * q + 1]) * sa * c.y);
        v[4 * q + 2] = __float_as_uint(__uint_as_float(v[4 * q + 2]) * sa * c.z);
        v[4 * q + 3] = __float_as_uint(__uint_as_float(v[4 * q + 3]) * sa * c.w);
    }
}

// 32 gate and 32 up columns -> 32 bf16 of h, packed in pairs.
__device__ __forceinline__ void swiglu_pack32(const uint32_t (&g)[32], const uint32_t (&u)[32], uint32_t (&packed)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
        packed[i] = pack_bf16x2(swiglu_f32(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                swiglu_f32(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
}

// 32 accumulator columns -> 32 bf16, packed in pairs.
__device__ __forceinline__ void pack32(const uint32_t (&v)[32], uint32_t (&packed)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
}

// A warp's 32 consecutive output rows x 32 bf16 (lane = row, 16 packed words each) stored through
// 2 KB of shared memory, so that a store instruction writes the 64 bytes of 8 whole rows (full
// 32-byte sectors) instead of 16 bytes of each of 32 rows (half sectors).  Lane l first writes
// its row to `stage` (its four 16-byte pieces XOR-swizzled by row: no bank conflicts either way),
// then stores piece l % 4 of row 8 j + l / 4 for j = 0..3; rows whose bit in `valid` is clear
// are skipped.  out0 = row 0, first column.  Warp-collective.
__device__ __forceinline__ void store_rows_staged(const uint32_t (&packed)[16], uint4* stage, int lane,
                                                  __nv_bfloat16* out0, long long ldo, uint32_t valid) {
    __syncwarp();                                   // the previous chunk's reads of stage are done
#pragma unroll
    for (int q = 0; q < 4; ++q)
        stage[lane * 4 + (q ^ ((lane >> 1) & 3))] =
            make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = 8 * j + (lane >> 2), q = lane & 3;
        const uint4 w = stage[r * 4 + (q ^ ((r >> 1) & 3))];
        if ((valid >> r) & 1u) reinterpret_cast<uint4*>(out0 + r * ldo)[q] = w;
    }
}

// store_rows_staged with one base pointer per row: lane l holds row l's (column 0) address in
// `row_ptr` (any value for rows whose bit in `valid` is clear); the 32 columns go to col0 onwards.
__device__ __forceinline__ void store_rows_staged_ptr(const uint32_t (&packed)[16], uint4* stage, int lane,
                                                      unsigned long long row_ptr, int col0, uint32_t valid) {
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q)
        stage[lane * 4 + (q ^ ((lane >> 1) & 3))] =
            make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = 8 * j + (lane >> 2), q = lane & 3;
        const uint4 w = stage[r * 4 + (q ^ ((r >> 1) & 3))];
        const unsigned long long p = __shfl_sync(0xffffffffu, row_ptr, r);
        if ((valid >> r) & 1u) reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p) + col0)[q] = w;
    }
}

// 32 gate and 32 up columns -> 32 bf16 of h, stored at dst (16-byte aligned).
__device__ __forceinline__ void swiglu_store32(const uint32_t (&g)[32], const uint32_t (&u)[32], __nv_bfloat16* dst) {
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        packed[i] = pack_bf16x2(swiglu_f32(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                swiglu_f32(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
}

// 32 accumulator columns -> 32 bf16 at dst (16-byte aligned).
__device__ __forceinline__ void store32(const uint32_t (&v)[32], __nv_bfloat16* dst) {
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
}

// F8: A and B are e4m3 (one byte per element, 128 K-elements per stage row of 128 bytes),
// tcgen05.mma kind::f8f6f4, and the epilogue applies the row and column scales.
template <int EPI, bool F8 = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB0b, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB1b,
                    const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.stages;
    uint8_t* sA = smem;
    uint8_t* sB = smem + S * GEMM_A_BYTES;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sB + S * p.b_slot);
    uint64_t* empty_bar = full_bar + S;
    uint64_t* tfull_bar = empty_bar + S;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* drain_bar = tempty_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar + s, 1);
            mbar_init(empty_bar + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar + a, 1);
            mbar_init(tempty_bar + a, 4);      // one arrival per epilogue warp
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA0);
        prefetch_tensormap(&tmB0);
        prefetch_tensormap(&tmA1);
        prefetch_tensormap(&tmB1);
        if (EPI == EPI_SWIGLU) {
            prefetch_tensormap(&tmB0b);
            prefetch_tensormap(&tmB1b);
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
            const uint64_t pol_b = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const GemmClass& c = p.cls[ti.cls];
                const CUtensorMap* mA = ti.cls ? &tmA1 : &tmA0;
                const CUtensorMap* mB = ti.cls ? &tmB1 : &tmB0;
                const CUtensorMap* mBb = ti.cls ? &tmB1b : &tmB0b;
                constexpr int KB = F8 ? 2 * GEMM_BK : GEMM_BK;   // K elements per 128-byte stage row
                const int nk = c.K / KB;
                const int k0 = ti.ks * c.K;
                const uint32_t bytes =
                    GEMM_A_BYTES + (EPI == EPI_SWIGLU ? 2u : 1u) * (uint32_t)c.b_tile_rows * GEMM_BK * 2u;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(empty_bar + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(full_bar + stage, bytes);
                    uint8_t* a_dst = sA + stage * GEMM_A_BYTES;
                    uint8_t* b_dst = sB + stage * p.b_slot;
                    tma_load_2d(a_dst, mA, full_bar + stage, k0 + kb * KB, ti.a_row, pol_a);
                    tma_load_2d(b_dst, mB, full_bar + stage, k0 + kb * KB, ti.b_row, pol_b);
                    if (EPI == EPI_SWIGLU)
                        tma_load_2d(b_dst + 128 * 128, mBb, full_bar + stage, k0 + kb * KB, ti.b_row, pol_b);
                    ++issued;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // another role gave up: let the copies already in flight land before exit
                const int n = issued < S ? issued : S;
                for (int i = 1; i <= n; ++i) {
                    const int q = issued - i;
                    mbar_wait(full_bar + (q % S), (uint32_t)((q / S) & 1), nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool any = false, ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
                const GemmClass& c = p.cls[ti.cls];
                const uint32_t idesc = F8 ? idesc_e4m3_f32(GEMM_BM, c.mma_n) : idesc_bf16_f32(GEMM_BM, c.mma_n);
                const int nk = c.K / (F8 ? 2 * GEMM_BK : GEMM_BK);
                if (!mbar_wait(tempty_bar + acc, acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GEMM_ACC_COLS);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(full_bar + stage, phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k_sw128(sA + stage * GEMM_A_BYTES);
                    const uint64_t bd = smem_desc_k_sw128(sB + stage * p.b_slot);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // 32 bytes of K per instruction (16 bf16 or 32 e4m3)
                        if (F8) umma_e4m3(d_tmem, ad + 2ull * kk, bd + 2ull * kk, idesc, (kb | kk) != 0);
                        else umma_bf16(d_tmem, ad + 2ull * kk, bd + 2ull * kk, idesc, (kb | kk) != 0);
                    }
                    umma_commit(empty_bar + stage);
                    any = true;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(tfull_bar + acc);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (any) {
                // every MMA issued by this thread has retired before TMEM is released
                umma_commit(drain_bar);
                mbar_wait(drain_bar, 0, nullptr);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int sub = warp & 3;                 // TMEM sub-partition of this warp
        const int row_in_tile = sub * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const TileInfo ti = gemm_decode_tile(p, t, routed_tiles);
            const GemmClass& c = p.cls[ti.cls];
            // tcgen05.ld is warp-collective: decide and proceed as a whole warp
            const bool ready = mbar_wait(tfull_bar + acc, acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t)(acc * GEMM_ACC_COLS) + ((uint32_t)(sub * 32) << 16);
            const long long orow = c.out_row0 + ti.a_row + row_in_tile;
            const bool row_ok = row_in_tile < ti.rows && orow >= 0 && orow < c.out_rows;

            // fp8: the A row's scale and the weight group's column scales
            float sa = 1.f;
            const float *sb = nullptr, *sb2 = nullptr;
            if (F8) {
                if (row_ok) sa = __ldg(c.a_scale + ti.a_row + row_in_tile);
                const long long wg = c.b_group_rows > 0 ? ti.b_row / c.b_group_rows : 0;
                sb = c.b_scale + wg * c.b_scale_stride;
                if (EPI == EPI_SWIGLU) sb2 = c.b_scale2 + wg * c.b_scale_stride;
            }
            if (EPI == EPI_SWIGLU) {
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(c.out) + orow * c.ldo;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t g[32], u[32];
                    __syncwarp();
                    tmem_ld_32cols(tbase + ch * 32, g);
                    tmem_ld_32cols(tbase + 128 + ch * 32, u);
                    tmem_ld_wait();
                    const int col0 = ti.n_idx * 128 + ch * 32;
                    if (row_ok && col0 < c.n_out) {
                        if (F8) {
                            scale_cols32(g, sa, sb + col0);
                            scale_cols32(u, sa, sb2 + col0);
                        }
                        swiglu_store32(g, u, out + col0);
                    }
                }
            } else if (EPI == EPI_STORE) {
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(c.out) + orow * c.ldo;
                if (c.row_addr && row_ok)
                    out = reinterpret_cast<__nv_bfloat16*>(__ldg(c.row_addr + ti.a_row + row_in_tile));
#pragma unroll 1
                for (int ch = 0; ch < c.mma_n / 32; ++ch) {
                    uint32_t v[32];
                    __syncwarp();
                    tmem_ld_32cols(tbase + ch * 32, v);
                    tmem_ld_wait();
                    const int col0 = ti.n_idx * c.b_tile_rows + ch * 32;
                    if (row_ok && col0 < c.n_out) {
                        if (F8) scale_cols32(v, sa, sb + col0);
                        store32(v, out + col0);
                    }
                }
            } else {  // EPI_LOGITS (K slice ks writes its partial sums split_stride further on)
                float* out = reinterpret_cast<float*>(c.out) + ti.ks * c.split_stride + orow * c.ldo;
                const bool vec_ok = (c.ldo & 3) == 0;
#pragma unroll 1
                for (int ch = 0; ch < c.mma_n / 32 + ((c.mma_n & 31) ? 1 : 0); ++ch) {
                    uint32_t v[32];
                    __syncwarp();
                    tmem_ld_32cols(tbase + ch * 32, v);
                    tmem_ld_wait();
                    const int col0 = ti.n_idx * c.b_tile_rows + ch * 32;
                    if (row_ok) {
                        if (vec_ok && col0 + 32 <= c.n_out) {
                            float4* dst = reinterpret_cast<float4*>(out + col0);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (col0 + i < c.n_out) out[col0 + i] = __uint_as_float(v[i]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();                     // every lane's tensor-memory reads are done
            if (lane == 0) mbar_arrive_relaxed(tempty_bar + acc);
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
