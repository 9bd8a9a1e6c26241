// grouped_gemm_pair.cuh - the grouped GEMM on CTA pairs (tcgen05 cta_group::2), for the
// expert FFN when experts hold many rows (prefill).
//
// Same products, group classes, tile walk and epilogues as grouped_gemm.cuh, but a tile is
// 256 rows x 256 columns computed by a cluster of two CTAs on two SMs:
//   - CTA r (r = 0, 1) loads rows [128 r, 128 r + 128) of the A tile and its half of the B
//     tile into its own shared memory (no multicast): for GEMM1 CTA 0 loads the W1 rows and
//     CTA 1 the same rows of W3; for GEMM2 CTA r loads W2 rows [n0 + 128 r, n0 + 128 r + 128).
//   - both CTAs' copies complete on the leader's (CTA 0) full barrier; one thread of the leader
//     issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), which reads both CTAs'
//     halves and accumulates rows [128 r, 128 r + 128) into CTA r's tensor memory.
//   - the leader's commits arrive on both CTAs' barriers (empty stage, accumulator full);
//     every epilogue warp of both CTAs (eight each) arrives once on the leader's
//     accumulator-empty barrier, after all its lanes' tensor-memory reads.
// Per SM this halves the B operand traffic of a 1-SM M = 128 tile and leaves room for a
// 6-stage ring (A 16 KB + B 16 KB per stage per CTA) and 16 KB of epilogue staging, through
// which each epilogue warp stores whole 64-byte pieces of 8 output rows at a time.
//
// Swapped tail tiles.  A group's last m-tile usually holds fewer than 256 rows; as an M = 256
// tile its MMAs would cost the same as a full one.  A tail tile of at most GemmParams::swap_max
// rows instead runs with the operands swapped, D^T = W * X^T: the weights are the M = 256 side (each
// CTA's 128 weight rows in the B slot of the stage) and the tile's tokens the N side (N = rows
// rounded up to 16, each CTA loading its N / 2 token rows in 32-row boxes into the A slot), so
// the MMA time follows the real row count.  TMEM then holds one weight row (output feature) per
// lane and one token per column.  For GEMM1 each CTA loads 64 rows of W1 and the same 64 rows of
// W3, so that a feature's gate (lanes 0-63) and up (lanes 64-127) values sit in the same CTA: the
// warps of lanes 64-127 pass their up values through shared memory to the warps of lanes 0-63,
// which apply SwiGLU.  Stores write one token row's 32 consecutive outputs (64 bytes) per warp
// instruction.
#pragma once

#include "grouped_gemm.cuh"

namespace moe {

constexpr int PAIR_BM = 256;                 // rows per pair tile
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_A_BYTES = 128 * GEMM_BK * 2;   // 16 KB per CTA
constexpr int PAIR_B_BYTES = 128 * GEMM_BK * 2;   // 16 KB per CTA
// warp 0 TMA, warp 1 MMA, warps 2..9 epilogue: two warps per TMEM lane quarter, each taking half
// of the accumulator's columns, so that the epilogue of one tile stays shorter than the next
// tile's MMAs even at the fp8 rate (twice the bf16 K per cycle).
constexpr int PAIR_EPI_WARPS = 8;
constexpr int PAIR_THREADS = 64 + 32 * PAIR_EPI_WARPS;
constexpr int PAIR_STAGE_OUT_BYTES = 2048;        // per epilogue warp: 32 rows x 32 bf16
constexpr int PAIR_SMEM_BYTES =
    PAIR_STAGES * (PAIR_A_BYTES + PAIR_B_BYTES) + PAIR_EPI_WARPS * PAIR_STAGE_OUT_BYTES + 1024 + 256;
constexpr int PAIR_SWAP_BOX_ROWS = 32;                      // token rows per TMA box of a swapped tile
constexpr int PAIR_SWAP_BOX_BYTES = PAIR_SWAP_BOX_ROWS * 128;

// Tensor maps only swapped tiles use.
struct PairSwapMaps {
    CUtensorMap a0, a1;     // the token rows of class 0 / class 1 in 32-row boxes
    CUtensorMap w0, w0b;    // GEMM1: W1 / W3 of class 0 in 64-row boxes
    CUtensorMap w1, w1b;    // GEMM1: W1 / W3 of class 1 in 64-row boxes
};


// Swapped tiles: a warp's 32 consecutive output columns (lane = column) x 32 tokens (vals[j] =
// token j, fp32 bits) as bf16, written through the warp's 2 KB staging slot so that each lane stores 16-byte
// pieces of token rows (a warp store covers 8 token rows x 64 bytes).  Token j goes to
// rowptr(j) + col0 (elements); tokens with j >= ntok are skipped.  Warp-collective.
template <typename RowPtr>
__device__ __forceinline__ void store_cols_transposed(const uint32_t (&vals)[32], __nv_bfloat16* stage, int lane,
                                                      int col0, int ntok, RowPtr rowptr) {
    __syncwarp();                                   // the slot's previous reads are done
#pragma unroll
    for (int j = 0; j < 32; ++j) stage[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(vals[j]));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int piece = lane + 32 * i, j = piece >> 2, q = piece & 3;
        if (j < ntok) {
            const uint4 w = reinterpret_cast<const uint4*>(stage + j * 32)[q];
            reinterpret_cast<uint4*>(rowptr(j) + col0)[q] = w;
        }
    }
}

// Tile walk with 256-row m-tiles (mprefix counts 256-row tiles per group).
__device__ __forceinline__ int pair_total_tiles(const GemmParams& p, int& routed_tiles) {
    routed_tiles = p.offsets ? __ldg(p.mprefix + p.E) * p.cls[0].ntiles : 0;
    const int dense = p.dense_rows ? ((p.dense_rows + PAIR_BM - 1) / PAIR_BM) * p.cls[1].ntiles : 0;
    return routed_tiles + dense;
}

struct PairTile {
    int cls;
    int a_row;   // first A row of the pair tile
    int rows;    // valid rows of the pair tile (<= 256)
    int group;
    int n_idx;
    bool swap;   // tail tile run with the operands swapped (tokens on the MMA's N side)
    int n_tok;   // swapped: MMA N = rows rounded up to 16
};

__device__ __forceinline__ PairTile pair_decode_tile(const GemmParams& p, int t, int routed_tiles, int swap_max) {
    PairTile ti;
    if (t < routed_tiles) {
        const GemmClass& c = p.cls[0];
        const int q = t / c.ntiles;
        int lo = 0, hi = p.E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(p.mprefix + mid) <= q) lo = mid; else hi = mid;
        }
        const int g = lo;
        const int mp = __ldg(p.mprefix + g);
        const int mt = __ldg(p.mprefix + g + 1) - mp;
        const int local = t - mp * c.ntiles;
        const int m = local % mt, n = local / mt;
        const int r0 = __ldg(p.offsets + g) + m * PAIR_BM;
        ti.cls = 0;
        ti.group = g;
        ti.a_row = r0;
        ti.rows = min(PAIR_BM, __ldg(p.offsets + g + 1) - r0);
        ti.n_idx = n;
    } else {
        const GemmClass& c = p.cls[1];
        const int mt = (p.dense_rows + PAIR_BM - 1) / PAIR_BM;
        const int local = t - routed_tiles;
        const int m = local % mt, n = local / mt;
        ti.cls = 1;
        ti.group = 0;
        ti.a_row = m * PAIR_BM;
        ti.rows = min(PAIR_BM, p.dense_rows - ti.a_row);
        ti.n_idx = n;
        (void)c;
    }
    ti.swap = ti.rows <= swap_max;
    ti.n_tok = (ti.rows + 15) & ~15;
    return ti;
}

// F8: e4m3 operands (128 K-elements per 128-byte stage row, kind::f8f6f4) and the epilogue
// applies the row and column scales of GemmClass.
template <int EPI, bool F8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmB0b, const __grid_constant__ CUtensorMap tmA1,
                         const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB1b,
                         const __grid_constant__ GemmParams p, const __grid_constant__ PairSwapMaps sw) {
    static_assert(EPI == EPI_SWIGLU || EPI == EPI_STORE, "pair tiles serve the expert GEMMs");
    const int swap_max = p.swap_max;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + PAIR_STAGES * PAIR_A_BYTES;
    uint8_t* sOut = sB + PAIR_STAGES * PAIR_B_BYTES;   // epilogue staging, one 2 KB slot per warp
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sOut + PAIR_EPI_WARPS * PAIR_STAGE_OUT_BYTES);
    uint64_t* empty_bar = full_bar + PAIR_STAGES;
    uint64_t* tfull_bar = empty_bar + PAIR_STAGES;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* drain_bar = tempty_bar + 2;
    uint64_t* xch_bar = drain_bar + 1;   // swapped GEMM1 tiles: 2 barriers per gate / up warp pair
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xch_bar + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0 = leader, 1 = peer
    const bool leader = rank == 0;
    const int pair_id = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < PAIR_STAGES; ++s) {
            mbar_init(full_bar + s, 1);      // leader: its producer's expect_tx; bytes of both CTAs
            mbar_init(empty_bar + s, 1);     // one multicast commit from the leader's MMA thread
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar + a, 1);     // one multicast commit
            mbar_init(tempty_bar + a, 2 * PAIR_EPI_WARPS);  // leader: one arrival per epilogue warp of 2 CTAs
        }
        mbar_init(drain_bar, 1);
        for (int i = 0; i < 8; ++i) mbar_init(xch_bar + i, 32);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA0);
        prefetch_tensormap(&tmB0);
        prefetch_tensormap(&tmB0b);
        prefetch_tensormap(&tmA1);
        prefetch_tensormap(&tmB1);
        prefetch_tensormap(&tmB1b);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, GEMM_TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // both CTAs' barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    int routed_tiles;
    const int total = pair_total_tiles(p, routed_tiles);

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_b = policy_evict_normal();
            const uint32_t full_leader0 = map_to_cta(full_bar, 0);
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = pair_id; t < total && ok; t += npairs) {
                const PairTile ti = pair_decode_tile(p, t, routed_tiles, swap_max);
                const GemmClass& c = p.cls[ti.cls];
                const CUtensorMap* mA = ti.cls ? &tmA1 : &tmA0;
                const CUtensorMap* mB;
                const int wg = ti.cls ? 0 : gemm_weight_group(p, ti.group);
                int b_row;
                if (EPI == EPI_SWIGLU) {       // CTA 0: W1 rows (gate), CTA 1: the same rows of W3 (up)
                    mB = ti.cls ? (leader ? &tmB1 : &tmB1b) : (leader ? &tmB0 : &tmB0b);
                    b_row = wg * c.b_group_rows + ti.n_idx * 128;
                } else {                       // CTA r: rows [n0 + 128 r, n0 + 128 r + 128) of W2
                    mB = ti.cls ? &tmB1 : &tmB0;
                    b_row = wg * c.b_group_rows + ti.n_idx * 256 + (int)rank * 128;
                }
                const int a_row = ti.a_row + (int)rank * 128;
                constexpr int KB = F8 ? 2 * GEMM_BK : GEMM_BK;
                const int nk = c.K / KB;
                // swapped tile: this CTA's N / 2 token rows in 32-row boxes, and its weight rows
                // (GEMM1: 64 rows of W1 and the same 64 rows of W3)
                const int half_tok = ti.n_tok >> 1;
                const int nld = ti.swap ? (half_tok + PAIR_SWAP_BOX_ROWS - 1) / PAIR_SWAP_BOX_ROWS : 0;
                const CUtensorMap* mT = ti.cls ? &sw.a1 : &sw.a0;
                const CUtensorMap* mW = ti.cls ? &sw.w1 : &sw.w0;
                const CUtensorMap* mWb = ti.cls ? &sw.w1b : &sw.w0b;
                const int t_row = ti.a_row + (int)rank * half_tok;
                const int w_row = wg * c.b_group_rows + ti.n_idx * 128 + (int)rank * 64;   // GEMM1 swapped
                const uint32_t tx = ti.swap ? 2u * (uint32_t)(PAIR_B_BYTES + nld * PAIR_SWAP_BOX_BYTES)
                                            : 2u * (PAIR_A_BYTES + PAIR_B_BYTES);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(empty_bar + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    const uint32_t fb = full_leader0 + (uint32_t)stage * 8u;
                    if (leader) mbar_arrive_expect_tx(full_bar + stage, tx);
                    if (!ti.swap) {
                        tma_load_2d_pair(sA + stage * PAIR_A_BYTES, mA, fb, kb * KB, a_row, pol_a);
                        tma_load_2d_pair(sB + stage * PAIR_B_BYTES, mB, fb, kb * KB, b_row, pol_b);
                    } else {
                        if (EPI == EPI_SWIGLU) {
                            tma_load_2d_pair(sB + stage * PAIR_B_BYTES, mW, fb, kb * KB, w_row, pol_b);
                            tma_load_2d_pair(sB + stage * PAIR_B_BYTES + 64 * 128, mWb, fb, kb * KB, w_row, pol_b);
                        } else {
                            tma_load_2d_pair(sB + stage * PAIR_B_BYTES, mB, fb, kb * KB, b_row, pol_b);
                        }
                        for (int i = 0; i < nld; ++i)
                            tma_load_2d_pair(sA + stage * PAIR_A_BYTES + i * PAIR_SWAP_BOX_BYTES, mT, fb, kb * KB,
                                             t_row + i * PAIR_SWAP_BOX_ROWS, pol_a);
                    }
                    ++issued;
                    if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok && leader) {
                // the leader's full barriers count both CTAs' copies; let those in flight land
                const int n = issued < PAIR_STAGES ? issued : PAIR_STAGES;
                for (int i = 1; i <= n; ++i) {
                    const int q = issued - i;
                    mbar_wait(full_bar + (q % PAIR_STAGES), (uint32_t)((q / PAIR_STAGES) & 1), nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer (leader only)
        if (lane == 0 && leader) {
            const uint32_t idesc = F8 ? idesc_e4m3_f32(PAIR_BM, 256) : idesc_bf16_f32(PAIR_BM, 256);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool any = false, ok = true;
            for (int t = pair_id; t < total && ok; t += npairs) {
                const PairTile ti = pair_decode_tile(p, t, routed_tiles, swap_max);
                const GemmClass& c = p.cls[ti.cls];
                const int nk = c.K / (F8 ? 2 * GEMM_BK : GEMM_BK);
                // swapped tile: A = the weights (B slot), B = the tokens (A slot), N = n_tok
                const uint32_t id = !ti.swap ? idesc
                                    : (F8 ? idesc_e4m3_f32(PAIR_BM, ti.n_tok) : idesc_bf16_f32(PAIR_BM, ti.n_tok));
                if (!mbar_wait(tempty_bar + acc, acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GEMM_ACC_COLS);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(full_bar + stage, phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t da = smem_desc_k_sw128(sA + stage * PAIR_A_BYTES);
                    const uint64_t db = smem_desc_k_sw128(sB + stage * PAIR_B_BYTES);
                    const uint64_t ad = ti.swap ? db : da;
                    const uint64_t bd = ti.swap ? da : db;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // 32 bytes of K per instruction
                        if (F8) umma_e4m3_pair(d_tmem, ad + 2ull * kk, bd + 2ull * kk, id, (kb | kk) != 0);
                        else umma_bf16_pair(d_tmem, ad + 2ull * kk, bd + 2ull * kk, id, (kb | kk) != 0);
                    }
                    umma_commit_pair(empty_bar + stage, 0x3);
                    any = true;
                    if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(tfull_bar + acc, 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (any) {
                umma_commit_pair(drain_bar, 0x1);
                mbar_wait(drain_bar, 0, nullptr);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue (both CTAs)
        const int sub = warp & 3;                 // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;         // which half of the columns it converts
        const int row_in_cta = sub * 32 + lane;
        const uint32_t tempty_leader0 = map_to_cta(tempty_bar, 0);
        uint4* stage = reinterpret_cast<uint4*>(sOut + (warp - 2) * PAIR_STAGE_OUT_BYTES);
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t xch_n = 0;         // swapped GEMM1 tiles: 16-token hand-overs so far (per pair)
        bool swap_ok = true;
        for (int t = pair_id; t < total && swap_ok; t += npairs) {
            const PairTile ti = pair_decode_tile(p, t, routed_tiles, swap_max);
            const GemmClass& c = p.cls[ti.cls];
            const bool ready = mbar_wait(tfull_bar + acc, acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t)(acc * GEMM_ACC_COLS) + ((uint32_t)(sub * 32) << 16);
            const int row_in_tile = (int)rank * 128 + row_in_cta;
            const long long orow = c.out_row0 + ti.a_row + row_in_tile;
            const bool row_ok = row_in_tile < ti.rows && orow >= 0 && orow < c.out_rows;
            // the warp's 32 rows are consecutive: out0 is its first row, valid has a bit per row
            // (with a row table: each lane's own row address instead)
            __nv_bfloat16* out0 = reinterpret_cast<__nv_bfloat16*>(c.out) + (orow - lane) * c.ldo;
            const uint32_t valid = __ballot_sync(0xffffffffu, row_ok);
            const unsigned long long row_ptr =
                (c.row_addr && row_ok) ? (unsigned long long)__ldg(c.row_addr + ti.a_row + row_in_tile) : 0ull;
            float sa = 1.f;                        // fp8: activation row scale, weight column scales
            const float *sb = nullptr, *sb2 = nullptr;
            if (F8) {
                if (row_ok) sa = __ldg(c.a_scale + ti.a_row + row_in_tile);
                const long long wg = ti.cls ? 0 : gemm_weight_group(p, ti.group);
                sb = c.b_scale + wg * c.b_scale_stride;
                if (EPI == EPI_SWIGLU) sb2 = c.b_scale2 + wg * c.b_scale_stride;
            }
            if (ti.swap) {
                // lane = weight row of this CTA, column j = token a_row + j; warp halves take
                // alternate 32-token chunks
                const int nch = (ti.n_tok + 31) >> 5;
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(c.out);
                if (EPI == EPI_SWIGLU) {
                    // lanes 0-63: gate of this CTA's 64 features, lanes 64-127: their up values; the
                    // warp of quarter q + 2 passes its up values to the warp of quarter q (same half)
                    // through the two warps' staging slots, tokens 0-15 / 16-31 of the chunk
                    const int q = sub & 1;
                    const bool up_warp = sub >= 2;
                    const int feat0 = ti.n_idx * 128 + (int)rank * 64 + q * 32;   // this warp's first feature
                    const int feat = feat0 + lane;
                    const bool feat_ok = feat < c.n_out;
                    __nv_bfloat16* own_stage =
                        reinterpret_cast<__nv_bfloat16*>(sOut + (warp - 2) * PAIR_STAGE_OUT_BYTES);
                    // the up warp's own staging slot: 16 tokens x 32 lanes of fp32; the pair's
                    // two barriers: values staged (up -> gate), values read (gate -> up)
                    float* st = reinterpret_cast<float*>(sOut + (q + 4 * half) * PAIR_STAGE_OUT_BYTES);
                    uint64_t* xch_staged = xch_bar + 2 * (q + 2 * half);
                    uint64_t* xch_read = xch_staged + 1;
                    float sg = 1.f, su = 1.f;
                    if (F8 && feat_ok) {
                        sg = __ldg(sb + feat);
                        su = __ldg(sb2 + feat);
                    }
#pragma unroll 1
                    for (int ch = half; ch < nch && swap_ok; ch += 2) {
                        uint32_t v[32];
                        __syncwarp();
                        tmem_ld_32cols(tbase + ch * 32, v);
                        tmem_ld_wait();
                        if (up_warp) {
                            // tokens 0-15, then 16-31 of the chunk through this warp's own slot
#pragma unroll
                            for (int part = 0; part < 2; ++part) {
                                if (!mbar_wait(xch_read, (xch_n & 1u) ^ 1u, abort_flag)) { swap_ok = false; break; }
#pragma unroll
                                for (int j = 0; j < 16; ++j) st[j * 32 + lane] = __uint_as_float(v[16 * part + j]);
                                mbar_arrive(xch_staged);
                                ++xch_n;
                            }
                        } else {
                            float u[32];
#pragma unroll
                            for (int part = 0; part < 2; ++part) {
                                if (!mbar_wait(xch_staged, xch_n & 1u, abort_flag)) { swap_ok = false; break; }
#pragma unroll
                                for (int j = 0; j < 16; ++j) u[16 * part + j] = st[j * 32 + lane];
                                mbar_arrive(xch_read);
                                ++xch_n;
                            }
                            if (!swap_ok) break;
                            // fp8: lane j holds token j's activation scale, broadcast per column
                            const float my_sa =
                                F8 ? __ldg(c.a_scale + ti.a_row + min(ch * 32 + lane, ti.rows - 1)) : 1.f;
#pragma unroll
                            for (int j = 0; j < 32; ++j) {     // h replaces the gate values in v
                                float g = __uint_as_float(v[j]), uu = u[j];
                                if (F8) {
                                    const float st_a = __shfl_sync(0xffffffffu, my_sa, j);
                                    g = g * st_a * sg;
                                    uu = uu * st_a * su;
                                }
                                v[j] = __float_as_uint(swiglu_f32(g, uu));
                            }
                            // this warp's 32 features are whole 64-byte pieces of h rows; the tile's
                            // features are all inside n_out (n_out is a multiple of 64)
                            const int ntok = min(32, ti.rows - ch * 32);
                            const long long row0 = c.out_row0 + ti.a_row + ch * 32;
                            if (feat0 < c.n_out)
                                store_cols_transposed(v, own_stage, lane, feat0, ntok, [&](int j) {
                                    return out + (row0 + j) * c.ldo;
                                });
                        }
                    }
                    // the up warp leaves its slot only once the last values were read from it
                    if (up_warp && swap_ok && !mbar_wait(xch_read, (xch_n & 1u) ^ 1u, abort_flag)) swap_ok = false;
                } else {
                    const int col0 = ti.n_idx * 256 + (int)rank * 128 + sub * 32;   // this warp's 32 columns
                    const float sc = (F8 && col0 + lane < c.n_out) ? __ldg(sb + col0 + lane) : 1.f;
                    __nv_bfloat16* own_stage =
                        reinterpret_cast<__nv_bfloat16*>(sOut + (warp - 2) * PAIR_STAGE_OUT_BYTES);
#pragma unroll 1
                    for (int ch = half; ch < nch; ch += 2) {
                        uint32_t v[32];
                        __syncwarp();
                        tmem_ld_32cols(tbase + ch * 32, v);
                        tmem_ld_wait();
                        if (F8) {
                            const float my_sa = __ldg(c.a_scale + ti.a_row + min(ch * 32 + lane, ti.rows - 1));
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                v[j] = __float_as_uint(__uint_as_float(v[j]) * __shfl_sync(0xffffffffu, my_sa, j) * sc);
                        }
                        const int ntok = min(32, ti.rows - ch * 32);
                        const int r0 = ti.a_row + ch * 32;
                        if (col0 < c.n_out) {
                            if (c.row_addr)
                                store_cols_transposed(v, own_stage, lane, col0, ntok, [&](int j) {
                                    return reinterpret_cast<__nv_bfloat16*>(__ldg(c.row_addr + r0 + j));
                                });
                            else
                                store_cols_transposed(v, own_stage, lane, col0, ntok, [&](int j) {
                                    return out + (c.out_row0 + r0 + j) * c.ldo;
                                });
                        }
                    }
                }
            } else if (EPI == EPI_SWIGLU) {
#pragma unroll 1
                for (int ch = 2 * half; ch < 2 * half + 2; ++ch) {
                    uint32_t g[32], u[32];
                    __syncwarp();
                    tmem_ld_32cols(tbase + ch * 32, g);
                    tmem_ld_32cols(tbase + 128 + ch * 32, u);
                    tmem_ld_wait();
                    const int col0 = ti.n_idx * 128 + ch * 32;
                    if (valid && col0 < c.n_out) {        // warp-uniform
                        if (F8) {
                            scale_cols32(g, sa, sb + col0);
                            scale_cols32(u, sa, sb2 + col0);
                        }
                        uint32_t packed[16];
                        swiglu_pack32(g, u, packed);
                        store_rows_staged(packed, stage, lane, out0 + col0, c.ldo, valid);
                    }
                }
            } else {
#pragma unroll 1
                for (int ch = 4 * half; ch < 4 * half + 4; ++ch) {
                    uint32_t v[32];
                    __syncwarp();
                    tmem_ld_32cols(tbase + ch * 32, v);
                    tmem_ld_wait();
                    const int col0 = ti.n_idx * 256 + ch * 32;
                    if (valid && col0 < c.n_out) {        // warp-uniform
                        if (F8) scale_cols32(v, sa, sb + col0);
                        uint32_t packed[16];
                        pack32(v, packed);
                        if (c.row_addr) store_rows_staged_ptr(packed, stage, lane, row_ptr, col0, valid);
                        else store_rows_staged(packed, stage, lane, out0 + col0, c.ldo, valid);
                    }
                }
            }
            if (!swap_ok) break;      // a hand-over wait gave up: the kernel is being abandoned
            tc_fence_before();
            __syncwarp();             // every lane's tensor-memory reads are done: one arrival per warp
            if (lane == 0) mbar_arrive_cluster_relaxed(tempty_leader0 + (uint32_t)acc * 8u);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    __syncthreads();
    cluster_sync_all();          // the leader's MMAs have drained; no remote arrivals remain
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, GEMM_TMEM_COLS);
    }
}

}  // namespace moe
