// moe_api.cu - the C ABI (include/moe.h): argument validation, TMA descriptors, launches.
//
// The host side never allocates device memory and never synchronises (except
// moe_get_error).  Every launch goes to the caller's stream.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "grouped_gemm.cuh"
#include "grouped_gemm_pair.cuh"
#include "grouped_gemm_w8.cuh"
#include "route_permute_combine.cuh"
#include "expert_cache.cuh"
#include "expert_parallel.cuh"
#include "act_quant.cuh"

namespace moe {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    bool ok = false;
    int sms = 0;
    bool gemm_attr = false;
    bool permute_attr = false;
    // expert cache: the stream the expert copies run on, and the fork / join events
    cudaStream_t copy_stream = nullptr;
    cudaEvent_t copy_fork = nullptr, copy_join = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& di = g_dev[dev];
    if (!di.init) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        di.ok = (major == 10 && minor == 0);
        di.init = true;
    }
    if (!di.ok) return MOE_ERR_DEVICE;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return MOE_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    *out = &di;
    return MOE_OK;
}

// The expert cache's copy stream and its fork / join events on this device (created once).
int copy_stream(DeviceInfo* di) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (di->copy_stream) return MOE_OK;
    if (cudaStreamCreateWithFlags(&di->copy_stream, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventCreateWithFlags(&di->copy_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&di->copy_join, cudaEventDisableTiming) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int check_shape(int T, int d, int E, int k, int f) {
    if (T < 1 || d < 64 || d % 64 || f < 64 || f % 64 || k < 1 || k > MAX_TOPK || E < k || E > 1024)
        return MOE_ERR_SHAPE;
    if ((long long)T * k >= (1ll << 31)) return MOE_ERR_SHAPE;
    return MOE_OK;
}

// 2-D bf16 tensor map [rows, inner], box [box_rows, 64], 128-byte swizzle, zero fill outside.
int make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)GEMM_BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// 2-D fp8 (byte) tensor map [rows, inner], box [box_rows, 64 bytes], unswizzled, zero fill outside.
// fp8 weights [rows, inner] bytes: boxes of box_rows rows x 64 bytes, 64-byte swizzle.
int make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {(cuuint32_t)GEMM_BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// e4m3 operands [rows, inner] bytes for the fp8 x fp8 GEMMs: boxes of box_rows rows x 128 bytes,
// 128-byte swizzle (the layout the K-major tcgen05 descriptors read).
int make_map_e4m3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

template <int EPI, bool F8 = false>
int launch_gemm(DeviceInfo* di, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& b0b,
                const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& b1b, GemmParams p,
                long long tiles_upper, cudaStream_t s) {
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        static bool attr_set[kMaxDevices][3] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (!attr_set[dev][EPI]) {
            if (cudaFuncSetAttribute(grouped_gemm_kernel<EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     GEMM_SMEM_MAX) != cudaSuccess)
                return MOE_ERR_CUDA;
            attr_set[dev][EPI] = true;
        }
    }
    if (tiles_upper <= 0) return MOE_OK;
    if (p.b_slot <= 0) p.b_slot = GEMM_B_BYTES;
    if (p.stages <= 0) {   // as many ring slots as fit
        p.stages = (GEMM_SMEM_MAX - 1024 - 256) / (GEMM_A_BYTES + p.b_slot);
        if (p.stages > GEMM_MAX_STAGES) p.stages = GEMM_MAX_STAGES;
    }
    const int smem = gemm_smem_bytes(p.stages, p.b_slot);
    const int grid = (int)(tiles_upper < di->sms ? tiles_upper : di->sms);
    grouped_gemm_kernel<EPI, F8><<<grid, GEMM_THREADS, smem, s>>>(a0, b0, b0b, a1, b1, b1b, p);
    return launch_status();
}

// K slices of the router GEMM when it has too few output tiles to occupy the GPU: slices
// double while the tile count stays under one CTA per SM of a B200 (148), each slice keeps
// >= 256 of K and the partial sums stay under 16 MB.  A pure function of the shapes, so the
// workspace size does not depend on the device.
// K slices of the router GEMM.  Precision first: one fp32 tensor-memory accumulation runs over at
// most ROUTER_MAX_K of the hidden dimension (measured on B200: over K = 4096 the logits drift up to
// 3.5e-5 from the exactly rounded sums, over K <= 1024 at most 5e-6); the slices are summed in fp32
// by the top-k kernel.  Then parallelism: small batches split further while the tiles do not fill
// the GPU.  Slices must be whole 64-element k-blocks of equal length.
constexpr int ROUTER_MAX_K = 512;
int router_ksplit(int T, int d, int E) {
    const long long tiles = (long long)((T + GEMM_BM - 1) / GEMM_BM) * ((E + 255) / 256);
    int ks = 1;
    while (d / ks > ROUTER_MAX_K && d % (GEMM_BK * ks * 2) == 0 && (long long)ks * 2 * T * E * 4 <= (512ll << 20))
        ks *= 2;
    while (tiles * ks * 2 <= 148 && d % (GEMM_BK * ks * 2) == 0 && d / (ks * 2) >= 256 &&
           (long long)ks * 2 * T * E * 4 <= (16ll << 20))
        ks *= 2;
    return ks;
}
size_t router_partial_bytes(int T, int d, int E) {
    const int ks = router_ksplit(T, d, E);
    return ks > 1 ? (size_t)ks * T * E * 4 : 0;
}

// Tail tiles of at most this many rows run with the operands swapped in the pair kernel (GEMM1,
// GEMM2); measured on the prefill workloads (same-box A/B): swapped SwiGLU tiles pay for their
// gate / up hand-over between warps, so GEMM1 swaps only short tails.
constexpr int kPairSwapMaxGemm1 = 64;
constexpr int kPairSwapMaxGemm2 = 128;

template <int EPI, bool F8 = false>
int launch_gemm_pair(DeviceInfo* di, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& b0b,
                     const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& b1b, const GemmParams& p,
                     const PairSwapMaps& sw, long long tiles_upper, cudaStream_t s) {
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        static bool attr_set[kMaxDevices][3] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (!attr_set[dev][EPI]) {
            if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     PAIR_SMEM_BYTES) != cudaSuccess)
                return MOE_ERR_CUDA;
            attr_set[dev][EPI] = true;
        }
    }
    if (tiles_upper <= 0) return MOE_OK;
    const long long pairs = di->sms / 2;
    const int grid = 2 * (int)(tiles_upper < pairs ? tiles_upper : pairs);
    GemmParams q = p;
    q.swap_max = EPI == EPI_SWIGLU ? kPairSwapMaxGemm1 : kPairSwapMaxGemm2;
    grouped_gemm_pair_kernel<EPI, F8><<<grid, PAIR_THREADS, PAIR_SMEM_BYTES, s>>>(a0, b0, b0b, a1, b1, b1b, q, sw);
    return launch_status();
}

// Pair (2-SM) tiles pay off when experts average at least one full 256-row tile.
bool use_pair_tiles(long long rows, int E) { return rows >= 256ll * E; }

// Tensor maps of the pair kernel's swapped tail tiles: the token rows of each class in 32-row
// boxes and (GEMM1) W1 / W3 of each class in 64-row boxes.  A null base leaves that map unused
// (its class has no rows, or the GEMM has no gate / up pair); it then copies another map.
// f8: e4m3 operands (128-byte K rows) instead of bf16.
int make_swap_maps(PairSwapMaps* m, bool f8, const void* t0, uint64_t k0, uint64_t rows0, const void* t1, uint64_t k1,
                   uint64_t rows1, const void* w1_0, const void* w3_0, uint64_t wrows0, const void* w1_1,
                   const void* w3_1, uint64_t wrows1) {
    memset(m, 0, sizeof(*m));
    auto mk = [&](CUtensorMap* d, const void* base, uint64_t inner, uint64_t rows, uint32_t box) {
        return f8 ? make_map_e4m3(d, base, inner, rows, box) : make_map(d, base, inner, rows, box);
    };
    int rc;
    if (t0 && (rc = mk(&m->a0, t0, k0, rows0, PAIR_SWAP_BOX_ROWS)) != MOE_OK) return rc;
    if (t1 && (rc = mk(&m->a1, t1, k1, rows1, PAIR_SWAP_BOX_ROWS)) != MOE_OK) return rc;
    if (w1_0 && (rc = mk(&m->w0, w1_0, k0, wrows0, 64)) != MOE_OK) return rc;
    if (w3_0 && (rc = mk(&m->w0b, w3_0, k0, wrows0, 64)) != MOE_OK) return rc;
    if (w1_1 && (rc = mk(&m->w1, w1_1, k1, wrows1, 64)) != MOE_OK) return rc;
    if (w3_1 && (rc = mk(&m->w1b, w3_1, k1, wrows1, 64)) != MOE_OK) return rc;
    if (!t0) { m->a0 = m->a1; m->w0 = m->w1; m->w0b = m->w1b; }
    if (!t1) { m->a1 = m->a0; m->w1 = m->w0; m->w1b = m->w0b; }
    return MOE_OK;
}

// ------------------------------------------------------------------ workspace layouts

struct LayerLayout {
    size_t off[12];
    size_t blk_cnt, rank_local, mprefix, h_shared, router_part, mp_hit, mp_miss;
    size_t total;
};

int permute_blocks(int T) { return (T + PERMUTE_TOKENS - 1) / PERMUTE_TOKENS; }

LayerLayout layer_layout(int T, int d, int E, int k, int f, int f_shared) {
    LayerLayout L;
    const size_t Tk = (size_t)T * k;
    size_t cur = 0;
    auto take = [&](size_t bytes) {
        size_t o = cur;
        cur = align256(cur + bytes);
        return o;
    };
    L.off[0] = take((size_t)T * E * 4);
    L.off[1] = take(Tk * 4);
    L.off[2] = take(Tk * 4);
    L.off[3] = take((size_t)E * 4);
    L.off[4] = take((size_t)E * 4);
    L.off[5] = take((size_t)(E + 1) * 4);
    L.off[6] = take(Tk * 4);
    L.off[7] = take(Tk * 4);
    L.off[8] = take(Tk * d * 2);
    L.off[9] = take(Tk * f * 2);
    L.off[10] = take(Tk * d * 2);
    L.off[11] = take(f_shared > 0 ? (size_t)T * d * 2 : 0);
    L.h_shared = take(f_shared > 0 ? (size_t)T * f_shared * 2 : 0);
    L.blk_cnt = take((size_t)permute_blocks(T) * E * 4);
    L.rank_local = take(Tk * 4);
    L.mprefix = take((size_t)(E + 1) * 4);
    L.router_part = take(router_partial_bytes(T, d, E));
    L.mp_hit = take((size_t)(E + 1) * 4);      // expert cache: tile prefixes of resident / loaded experts
    L.mp_miss = take((size_t)(E + 1) * 4);
    L.total = cur;
    return L;
}

// fp8 activations of the fp8 x fp8 layer, after the layer workspace: the permuted rows and h
// (routed), x and h of the shared expert, each as e4m3 codes plus one fp32 scale per row.
struct A8Layout {
    size_t xq, sx, hq, sh, xqs, sxs, hqs, shs, total;
};

A8Layout a8_layout(size_t base, int T, int d, int k, int f, int f_shared) {
    A8Layout A;
    const size_t Tk = (size_t)T * k;
    size_t cur = align256(base);
    auto take = [&](size_t bytes) {
        size_t o = cur;
        cur = align256(cur + bytes);
        return o;
    };
    A.xq = take(Tk * d);
    A.sx = take(Tk * 4);
    A.hq = take(Tk * f);
    A.sh = take(Tk * 4);
    A.xqs = take(f_shared > 0 ? (size_t)T * d : 0);
    A.sxs = take(f_shared > 0 ? (size_t)T * 4 : 0);
    A.hqs = take(f_shared > 0 ? (size_t)T * f_shared : 0);
    A.shs = take(f_shared > 0 ? (size_t)T * 4 : 0);
    A.total = cur;
    return A;
}

// scratch used by moe_permute: blk_cnt + rank_local + mprefix
size_t permute_scratch_bytes(int T, int E, int k, size_t* o_blk, size_t* o_rank, size_t* o_mp) {
    size_t cur = 0;
    *o_blk = cur;
    cur = align256(cur + (size_t)permute_blocks(T) * E * 4);
    *o_rank = cur;
    cur = align256(cur + (size_t)T * k * 4);
    *o_mp = cur;
    cur = align256(cur + (size_t)(E + 1) * 4);
    return cur;
}

// ------------------------------------------------------------------ stage launchers

// Router logits.  ks == 1: writes `logits` [T,E]; ks > 1: writes ks partial sums into
// `partials` ([ks][T][E]), which the top-k kernel adds up.
int run_router_gemm(DeviceInfo* di, const moe_bf16* x, const moe_bf16* Wg, int T, int d, int E, float* logits,
                    float* partials, int ks, cudaStream_t s) {
    const int npad = E <= 256 ? ((E + 15) / 16) * 16 : 256;
    CUtensorMap a, b;
    int rc;
    if ((rc = make_map(&a, x, d, T, GEMM_BM)) != MOE_OK) return rc;
    if ((rc = make_map(&b, Wg, d, E, npad)) != MOE_OK) return rc;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    GemmClass& c = p.cls[1];
    c.K = d / ks;
    c.n_out = E;
    c.ntiles = (E + npad - 1) / npad;
    c.b_group_rows = 0;
    c.b_tile_rows = npad;
    c.mma_n = npad;
    c.out = ks > 1 ? partials : logits;
    c.ldo = E;
    c.out_row0 = 0;
    c.out_rows = T;
    c.ksplit = ks;
    c.split_stride = (long long)T * E;
    p.cls[0] = c;
    p.offsets = nullptr;
    p.mprefix = nullptr;
    p.E = E;
    p.dense_rows = T;
    p.b_slot = npad * GEMM_BK * 2;      // a narrow B tile leaves room for more ring slots
    p.stages = 0;
    const long long tiles = (long long)((T + GEMM_BM - 1) / GEMM_BM) * c.ntiles * ks;
    return launch_gemm<EPI_LOGITS>(di, a, b, b, a, b, b, p, tiles, s);
}

// Top-k on `logits` ([T,E]); with nsplit > 1 `logits` holds nsplit partial sums [nsplit][T][E]
// that are added first (their sums go to logits_out).
int run_topk(const float* logits, int nsplit, float* logits_out, const float* bias, int T, int E, int k,
             int32_t* idx, float* w, cudaStream_t s) {
    const int blocks = (T + 7) / 8;
    const int epl = (E + 31) / 32;
    const long long st = (long long)T * E;
#define MOE_TOPK(EPL) topk_softmax_kernel<EPL><<<blocks, 256, 0, s>>>(logits, nsplit, st, logits_out, bias, T, E, k, idx, w)
    if (epl <= 1) MOE_TOPK(1);
    else if (epl <= 2) MOE_TOPK(2);
    else if (epl <= 4) MOE_TOPK(4);
    else if (epl <= 8) MOE_TOPK(8);
    else if (epl <= 16) MOE_TOPK(16);
    else MOE_TOPK(32);
#undef MOE_TOPK
    return launch_status();
}

int run_permute(DeviceInfo* di, const moe_bf16* x, const int32_t* idx, int T, int d, int E, int k, long long C,
                int32_t* counts_raw, int32_t* counts, int32_t* offsets, int32_t* dest, int32_t* src_token,
                moe_bf16* x_perm, int32_t* blk_cnt, int32_t* rank_local, int32_t* mprefix, cudaStream_t s,
                int tile_rows = GEMM_BM, const int32_t* fill_base = nullptr, bool counts_only = false,
                bool gather = true) {
    const int nb = permute_blocks(T);
    const size_t smem = (size_t)(PERMUTE_WARPS * E + PERMUTE_TOKENS * k) * sizeof(int);
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!di->permute_attr) {
            if (cudaFuncSetAttribute(permute_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (PERMUTE_WARPS * 1024 + PERMUTE_TOKENS * MAX_TOPK) * (int)sizeof(int)) !=
                cudaSuccess)
                return MOE_ERR_CUDA;
            di->permute_attr = true;
        }
    }
    permute_count_kernel<<<nb, PERMUTE_TOKENS, smem, s>>>(idx, T, E, k, blk_cnt, rank_local);
    permute_scan_kernel<<<1, 1024, 0, s>>>(blk_cnt, nb, E, C, fill_base, counts_raw, counts, offsets, mprefix,
                                           tile_rows);
    if (counts_only) return launch_status();
    permute_scatter_kernel<<<nb, PERMUTE_TOKENS, 0, s>>>(idx, rank_local, blk_cnt, offsets, T, E, k, C, fill_base, dest,
                                                          src_token);
    if (!gather) return launch_status();   // the caller moves x's rows itself (dest / src_token)
    const long long chunks = (long long)T * (d / 8);
    gather_rows_kernel<<<(unsigned)((chunks + 255) / 256), 256, 0, s>>>(reinterpret_cast<const uint4*>(x), dest, T,
                                                                         d, k, reinterpret_cast<uint4*>(x_perm));
    return launch_status();
}

// Both grouped GEMMs of the expert FFN.  Class 0: routed experts on x_perm rows given by
// offsets/mprefix.  Class 1 (optional): the shared expert on all T rows of x.
struct FfnArgs {
    const moe_bf16* x_perm;
    const int32_t* offsets;
    const int32_t* mprefix;
    int max_rows, E, d, f;
    const moe_bf16 *W1, *W3, *W2;
    moe_bf16 *h, *y_perm;
    // shared expert (f_shared = 0: none)
    const moe_bf16* x;
    int T, f_shared;
    const moe_bf16 *W1s, *W3s, *W2s;
    moe_bf16 *h_shared, *y_shared;
    bool pair;   // 2-SM tiles (mprefix counts 256-row tiles) instead of 1-SM tiles (128 rows)
    const int32_t* group_map;   // routed group -> weight group (expert cache slots), nullptr = identity
    int w_groups;               // weight groups in W1/W3/W2 (0 = E)
    const long long* y_row_addr;  // nullable: GEMM2 stores routed row r at this byte address (fused return)
};

inline uint64_t weight_groups(const FfnArgs& a) { return (uint64_t)(a.w_groups ? a.w_groups : a.E); }

int run_expert_ffn(DeviceInfo* di, const FfnArgs& a, cudaStream_t s, cudaEvent_t ev_down = nullptr) {
    const bool shared = a.f_shared > 0;
    const bool routed = a.max_rows > 0;
    int rc;
    // ---- GEMM1: h = silu(x W1^T) * (x W3^T)
    {
        CUtensorMap A0, B0, B0b, A1, B1, B1b;
        if (routed) {
            if ((rc = make_map(&A0, a.x_perm, a.d, a.max_rows, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&B0, a.W1, a.d, weight_groups(a) * a.f, 128)) != MOE_OK) return rc;
            if ((rc = make_map(&B0b, a.W3, a.d, weight_groups(a) * a.f, 128)) != MOE_OK) return rc;
        }
        if (shared) {
            if ((rc = make_map(&A1, a.x, a.d, a.T, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&B1, a.W1s, a.d, a.f_shared, 128)) != MOE_OK) return rc;
            if ((rc = make_map(&B1b, a.W3s, a.d, a.f_shared, 128)) != MOE_OK) return rc;
        }
        if (!routed) { A0 = A1; B0 = B1; B0b = B1b; }
        if (!shared) { A1 = A0; B1 = B0; B1b = B0b; }
        GemmParams p;
        memset(&p, 0, sizeof(p));
        GemmClass& c0 = p.cls[0];
        c0.K = a.d; c0.n_out = a.f; c0.ntiles = (a.f + 127) / 128; c0.b_group_rows = a.f; c0.b_tile_rows = 128;
        c0.mma_n = 256; c0.out = a.h; c0.ldo = a.f; c0.out_row0 = 0; c0.out_rows = a.max_rows;
        GemmClass& c1 = p.cls[1];
        c1.K = a.d; c1.n_out = a.f_shared; c1.ntiles = (a.f_shared + 127) / 128; c1.b_group_rows = 0;
        c1.b_tile_rows = 128; c1.mma_n = 256; c1.out = a.h_shared; c1.ldo = a.f_shared; c1.out_row0 = 0;
        c1.out_rows = a.T;
        c0.ksplit = c1.ksplit = 1;
        p.offsets = routed ? a.offsets : nullptr;
        p.mprefix = a.mprefix;
        p.E = a.E;
        p.dense_rows = shared ? a.T : 0;
        p.b_slot = GEMM_B_BYTES;
        p.group_map = a.group_map;
        p.stages = GEMM_STAGES;
        long long tiles = 0;
        const int bm = a.pair ? PAIR_BM : GEMM_BM;
        if (routed) tiles += ((long long)(a.max_rows + bm - 1) / bm + a.E) * c0.ntiles;
        if (shared) tiles += (long long)((a.T + bm - 1) / bm) * c1.ntiles;
        PairSwapMaps sw;
        if (a.pair && (rc = make_swap_maps(&sw, false, routed ? a.x_perm : nullptr, a.d, a.max_rows,
                                           shared ? a.x : nullptr, a.d, a.T, routed ? a.W1 : nullptr,
                                           routed ? a.W3 : nullptr, weight_groups(a) * a.f, shared ? a.W1s : nullptr,
                                           shared ? a.W3s : nullptr, a.f_shared)) != MOE_OK)
            return rc;
        rc = a.pair ? launch_gemm_pair<EPI_SWIGLU>(di, A0, B0, B0b, A1, B1, B1b, p, sw, tiles, s)
                    : launch_gemm<EPI_SWIGLU>(di, A0, B0, B0b, A1, B1, B1b, p, tiles, s);
        if (rc != MOE_OK) return rc;
    }
    if (ev_down && cudaEventRecord(ev_down, s) != cudaSuccess) return MOE_ERR_CUDA;
    // ---- GEMM2: y = h W2^T
    {
        CUtensorMap A0, B0, A1, B1;
        if (routed) {
            if ((rc = make_map(&A0, a.h, a.f, a.max_rows, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&B0, a.W2, a.f, weight_groups(a) * a.d, a.pair ? 128 : 256)) != MOE_OK) return rc;
        }
        if (shared) {
            if ((rc = make_map(&A1, a.h_shared, a.f_shared, a.T, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&B1, a.W2s, a.f_shared, a.d, a.pair ? 128 : 256)) != MOE_OK) return rc;
        }
        if (!routed) { A0 = A1; B0 = B1; }
        if (!shared) { A1 = A0; B1 = B0; }
        GemmParams p;
        memset(&p, 0, sizeof(p));
        GemmClass& c0 = p.cls[0];
        c0.K = a.f; c0.n_out = a.d; c0.ntiles = (a.d + 255) / 256; c0.b_group_rows = a.d; c0.b_tile_rows = 256;
        c0.mma_n = 256; c0.out = a.y_perm; c0.ldo = a.d; c0.out_row0 = 0; c0.out_rows = a.max_rows;
        c0.row_addr = a.y_row_addr;
        GemmClass& c1 = p.cls[1];
        c1.K = a.f_shared; c1.n_out = a.d; c1.ntiles = (a.d + 255) / 256; c1.b_group_rows = 0; c1.b_tile_rows = 256;
        c1.mma_n = 256; c1.out = a.y_shared; c1.ldo = a.d; c1.out_row0 = 0; c1.out_rows = a.T;
        c0.ksplit = c1.ksplit = 1;
        p.offsets = routed ? a.offsets : nullptr;
        p.mprefix = a.mprefix;
        p.E = a.E;
        p.dense_rows = shared ? a.T : 0;
        p.b_slot = GEMM_B_BYTES;
        p.group_map = a.group_map;
        p.stages = GEMM_STAGES;
        long long tiles = 0;
        const int bm = a.pair ? PAIR_BM : GEMM_BM;
        if (routed) tiles += ((long long)(a.max_rows + bm - 1) / bm + a.E) * c0.ntiles;
        if (shared) tiles += (long long)((a.T + bm - 1) / bm) * c1.ntiles;
        PairSwapMaps sw;
        if (a.pair && (rc = make_swap_maps(&sw, false, routed ? a.h : nullptr, a.f, a.max_rows,
                                           shared ? a.h_shared : nullptr, a.f_shared, a.T, nullptr, nullptr, 0,
                                           nullptr, nullptr, 0)) != MOE_OK)
            return rc;
        rc = a.pair ? launch_gemm_pair<EPI_STORE>(di, A0, B0, B0, A1, B1, B1, p, sw, tiles, s)
                    : launch_gemm<EPI_STORE>(di, A0, B0, B0, A1, B1, B1, p, tiles, s);
        if (rc != MOE_OK) return rc;
    }
    return MOE_OK;
}

// fp8 e4m3 expert weights with fp32 row scales (routed: W1q/W3q [E,f,d], s1/s3 [E,f], W2q [E,d,f],
// s2 [E,d]; shared: W1sq/W3sq [f_s,d], s1s/s3s [f_s], W2sq [d,f_s], s2s [d]).
struct W8Weights {
    const uint8_t *W1q, *W3q, *W2q, *W1sq, *W3sq, *W2sq;
    const float *s1, *s3, *s2, *s1s, *s3s, *s2s;
};

template <int EPI>
int launch_gemm_w8(DeviceInfo* di, const CUtensorMap* maps, const GemmParams& p, const W8Scales& sc,
                   long long tiles_upper, cudaStream_t s) {
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        static bool attr_set[kMaxDevices][3] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (!attr_set[dev][EPI]) {
            if (cudaFuncSetAttribute(grouped_gemm_w8_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     W8_SMEM_BYTES) != cudaSuccess)
                return MOE_ERR_CUDA;
            attr_set[dev][EPI] = true;
        }
    }
    if (tiles_upper <= 0) return MOE_OK;
    const int grid = (int)(tiles_upper < di->sms ? tiles_upper : di->sms);
    grouped_gemm_w8_kernel<EPI><<<grid, W8_THREADS, W8_SMEM_BYTES, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                                        maps[5], maps[6], maps[7], p, sc);
    return launch_status();
}

int run_expert_ffn_w8(DeviceInfo* di, const FfnArgs& a, const W8Weights& q, cudaStream_t s, cudaEvent_t ev_down) {
    const bool shared = a.f_shared > 0;
    const bool routed = a.max_rows > 0;
    int rc;
    // ---- GEMM1 (maps: A, A32, W1q, W3q for routed, then shared)
    {
        CUtensorMap m[8];
        if (routed) {
            if ((rc = make_map(&m[0], a.x_perm, a.d, a.max_rows, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&m[1], a.x_perm, a.d, a.max_rows, 32)) != MOE_OK) return rc;
            if ((rc = make_map_u8(&m[2], q.W1q, a.d, weight_groups(a) * a.f, 128)) != MOE_OK) return rc;
            if ((rc = make_map_u8(&m[3], q.W3q, a.d, weight_groups(a) * a.f, 128)) != MOE_OK) return rc;
        }
        if (shared) {
            if ((rc = make_map(&m[4], a.x, a.d, a.T, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&m[5], a.x, a.d, a.T, 32)) != MOE_OK) return rc;
            if ((rc = make_map_u8(&m[6], q.W1sq, a.d, a.f_shared, 128)) != MOE_OK) return rc;
            if ((rc = make_map_u8(&m[7], q.W3sq, a.d, a.f_shared, 128)) != MOE_OK) return rc;
        }
        for (int i = 0; i < 4; ++i) {
            if (!routed) m[i] = m[i + 4];
            if (!shared) m[i + 4] = m[i];
        }
        GemmParams p;
        memset(&p, 0, sizeof(p));
        GemmClass& c0 = p.cls[0];
        c0.K = a.d; c0.n_out = a.f; c0.ntiles = (a.f + 127) / 128; c0.b_group_rows = a.f; c0.b_tile_rows = 128;
        c0.mma_n = 256; c0.out = a.h; c0.ldo = a.f; c0.out_row0 = 0; c0.out_rows = a.max_rows; c0.ksplit = 1;
        GemmClass& c1 = p.cls[1];
        c1.K = a.d; c1.n_out = a.f_shared; c1.ntiles = (a.f_shared + 127) / 128; c1.b_group_rows = 0;
        c1.b_tile_rows = 128; c1.mma_n = 256; c1.out = a.h_shared; c1.ldo = a.f_shared; c1.out_row0 = 0;
        c1.out_rows = a.T; c1.ksplit = 1;
        p.offsets = routed ? a.offsets : nullptr;
        p.mprefix = a.mprefix;
        p.E = a.E;
        p.dense_rows = shared ? a.T : 0;
        p.group_map = a.group_map;   // scales follow: the epilogue finds them by the mapped weight row
        W8Scales sc;
        memset(&sc, 0, sizeof(sc));
        sc.s0[0] = q.s1; sc.s1[0] = q.s3; sc.group_stride[0] = a.f;
        sc.s0[1] = shared ? q.s1s : q.s1; sc.s1[1] = shared ? q.s3s : q.s3; sc.group_stride[1] = 0;
        long long tiles = 0;
        if (routed) tiles += ((long long)(a.max_rows + GEMM_BM - 1) / GEMM_BM + a.E) * c0.ntiles;
        if (shared) tiles += (long long)((a.T + GEMM_BM - 1) / GEMM_BM) * c1.ntiles;
        if ((rc = launch_gemm_w8<EPI_SWIGLU>(di, m, p, sc, tiles, s)) != MOE_OK) return rc;
    }
    if (ev_down && cudaEventRecord(ev_down, s) != cudaSuccess) return MOE_ERR_CUDA;
    // ---- GEMM2 (maps: A = h, A32, W2q; second W map unused)
    {
        CUtensorMap m[8];
        if (routed) {
            if ((rc = make_map(&m[0], a.h, a.f, a.max_rows, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&m[1], a.h, a.f, a.max_rows, 32)) != MOE_OK) return rc;
            if ((rc = make_map_u8(&m[2], q.W2q, a.f, weight_groups(a) * a.d, 256)) != MOE_OK) return rc;
            m[3] = m[2];
        }
        if (shared) {
            if ((rc = make_map(&m[4], a.h_shared, a.f_shared, a.T, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map(&m[5], a.h_shared, a.f_shared, a.T, 32)) != MOE_OK) return rc;
            if ((rc = make_map_u8(&m[6], q.W2sq, a.f_shared, a.d, 256)) != MOE_OK) return rc;
            m[7] = m[6];
        }
        for (int i = 0; i < 4; ++i) {
            if (!routed) m[i] = m[i + 4];
            if (!shared) m[i + 4] = m[i];
        }
        GemmParams p;
        memset(&p, 0, sizeof(p));
        GemmClass& c0 = p.cls[0];
        c0.K = a.f; c0.n_out = a.d; c0.ntiles = (a.d + 255) / 256; c0.b_group_rows = a.d; c0.b_tile_rows = 256;
        c0.mma_n = 256; c0.out = a.y_perm; c0.ldo = a.d; c0.out_row0 = 0; c0.out_rows = a.max_rows; c0.ksplit = 1;
        GemmClass& c1 = p.cls[1];
        c1.K = a.f_shared; c1.n_out = a.d; c1.ntiles = (a.d + 255) / 256; c1.b_group_rows = 0; c1.b_tile_rows = 256;
        c1.mma_n = 256; c1.out = a.y_shared; c1.ldo = a.d; c1.out_row0 = 0; c1.out_rows = a.T; c1.ksplit = 1;
        p.offsets = routed ? a.offsets : nullptr;
        p.mprefix = a.mprefix;
        p.E = a.E;
        p.dense_rows = shared ? a.T : 0;
        p.group_map = a.group_map;   // scales follow: the epilogue finds them by the mapped weight row
        W8Scales sc;
        memset(&sc, 0, sizeof(sc));
        sc.s0[0] = q.s2; sc.group_stride[0] = a.d;
        sc.s0[1] = shared ? q.s2s : q.s2; sc.group_stride[1] = 0;
        long long tiles = 0;
        if (routed) tiles += ((long long)(a.max_rows + GEMM_BM - 1) / GEMM_BM + a.E) * c0.ntiles;
        if (shared) tiles += (long long)((a.T + GEMM_BM - 1) / GEMM_BM) * c1.ntiles;
        if ((rc = launch_gemm_w8<EPI_STORE>(di, m, p, sc, tiles, s)) != MOE_OK) return rc;
    }
    return MOE_OK;
}

// Both expert GEMMs with fp8 weights and fp8 activations: each token row of x is quantised once
// and its codes written to its k permuted rows (dest) and, with a shared expert, to its own row;
// h rows after GEMM1; the grouped GEMMs run kind::f8f6f4 and scale each accumulator by its
// activation row scale and weight row scale.
struct A8Bufs {
    uint8_t *xq, *hq, *xqs, *hqs;
    float *sx, *sh, *sxs, *shs;
    const int32_t* dest;        // [T, k] permuted row of each assignment, -1 = dropped
    const int32_t* src_token;   // [T k] token of each permuted row (for rows too long to hold)
    int k;
};

int run_quant_rows(const void* src, const int32_t* gather, const int32_t* n_rows, int rows, int K, uint8_t* dst,
                   float* scale, cudaStream_t s) {
    if (rows <= 0) return MOE_OK;
    quant_rows_e4m3_kernel<<<(rows + 7) / 8, 256, 0, s>>>(static_cast<const uint4*>(src), gather, n_rows, rows, K,
                                                          reinterpret_cast<uint2*>(dst), scale);
    return launch_status();
}

// The register-held quantiser for rows of up to 16384 elements: a warp per row up to 2048
// elements, 128 threads up to 8192, 256 beyond; returns false (nothing launched) for longer rows.
bool run_quant_blk(const void* src, const int32_t* n_rows, int rows, int K, const int32_t* dest, int k, uint8_t* dst,
                   float* scale, uint8_t* dst_tok, float* scale_tok, cudaStream_t s) {
    const int chunks = K / 8;
    const uint4* x = static_cast<const uint4*>(src);
    uint2* d = reinterpret_cast<uint2*>(dst);
    uint2* dt = reinterpret_cast<uint2*>(dst_tok);
#define MOE_QUANT(TPR, C)                                                                                    \
    quant_rows_e4m3_reg_kernel<TPR, C><<<(unsigned)(((long long)rows * TPR + QUANT_CTA - 1) / QUANT_CTA),      \
                                         QUANT_CTA, 0, s>>>(x, n_rows, rows, K, dest, k, d, scale, dt, scale_tok)
    if (chunks <= 32 * 2) MOE_QUANT(32, 2);
    else if (chunks <= 32 * 4) MOE_QUANT(32, 4);
    else if (chunks <= 32 * 8) MOE_QUANT(32, 8);
    else if (chunks <= 128 * 4) MOE_QUANT(128, 4);
    else if (chunks <= 128 * 8) MOE_QUANT(128, 8);
    else if (chunks <= 256 * 8) MOE_QUANT(256, 8);
    else return false;
#undef MOE_QUANT
    return true;
}

// h rows [0, *n_rows) of a [rows, K] buffer -> e4m3 rows + scales.  Rows of up to 2048
// elements take the two-pass warp-per-row kernel: its 28 registers keep 64 warps per SM busy
// with the correctly rounded divisions, and its second pass over a row hits L2 (measured faster
// than holding the row in registers for K = 1536 and 2048); longer rows are read once.
int run_quant_h(const void* h, const int32_t* n_rows, int rows, int K, uint8_t* dst, float* scale, cudaStream_t s) {
    if (rows <= 0) return MOE_OK;
    if (K <= 2048 || !run_quant_blk(h, n_rows, rows, K, nullptr, 0, dst, scale, nullptr, nullptr, s))
        return run_quant_rows(h, nullptr, n_rows, rows, K, dst, scale, s);
    return launch_status();
}

int run_expert_ffn_a8(DeviceInfo* di, const FfnArgs& a, const W8Weights& q, const A8Bufs& b, cudaStream_t s,
                      cudaEvent_t ev_down, cudaEvent_t ev_gemm1, cudaEvent_t ev_gemm2) {
    const bool shared = a.f_shared > 0;
    const bool routed = a.max_rows > 0;
    const int32_t* n_routed = routed ? a.offsets + a.E : nullptr;   // kept rows (device)
    int rc;
    // x: every token row quantised once, its codes written to its permuted rows (and its own
    // row for the shared expert)
    if (routed && run_quant_blk(a.x, nullptr, a.T, a.d, b.dest, b.k, b.xq, b.sx, shared ? b.xqs : nullptr,
                                shared ? b.sxs : nullptr, s)) {
        if ((rc = launch_status()) != MOE_OK) return rc;
    } else {
        if (routed && (rc = run_quant_rows(a.x, b.src_token, n_routed, a.max_rows, a.d, b.xq, b.sx, s)) != MOE_OK)
            return rc;
        if (shared && (rc = run_quant_h(a.x, nullptr, a.T, a.d, b.xqs, b.sxs, s)) != MOE_OK) return rc;
    }
    if (ev_gemm1 && cudaEventRecord(ev_gemm1, s) != cudaSuccess) return MOE_ERR_CUDA;
    // ---- GEMM1: h = silu(s_x s1 (xq W1q^T)) * (s_x s3 (xq W3q^T))
    {
        CUtensorMap A0, B0, B0b, A1, B1, B1b;
        if (routed) {
            if ((rc = make_map_e4m3(&A0, b.xq, a.d, a.max_rows, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map_e4m3(&B0, q.W1q, a.d, weight_groups(a) * a.f, 128)) != MOE_OK) return rc;
            if ((rc = make_map_e4m3(&B0b, q.W3q, a.d, weight_groups(a) * a.f, 128)) != MOE_OK) return rc;
        }
        if (shared) {
            if ((rc = make_map_e4m3(&A1, b.xqs, a.d, a.T, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map_e4m3(&B1, q.W1sq, a.d, a.f_shared, 128)) != MOE_OK) return rc;
            if ((rc = make_map_e4m3(&B1b, q.W3sq, a.d, a.f_shared, 128)) != MOE_OK) return rc;
        }
        if (!routed) { A0 = A1; B0 = B1; B0b = B1b; }
        if (!shared) { A1 = A0; B1 = B0; B1b = B0b; }
        GemmParams p;
        memset(&p, 0, sizeof(p));
        GemmClass& c0 = p.cls[0];
        c0.K = a.d; c0.n_out = a.f; c0.ntiles = (a.f + 127) / 128; c0.b_group_rows = a.f; c0.b_tile_rows = 128;
        c0.mma_n = 256; c0.out = a.h; c0.ldo = a.f; c0.out_row0 = 0; c0.out_rows = a.max_rows;
        c0.a_scale = b.sx; c0.b_scale = q.s1; c0.b_scale2 = q.s3; c0.b_scale_stride = a.f;
        GemmClass& c1 = p.cls[1];
        c1.K = a.d; c1.n_out = a.f_shared; c1.ntiles = (a.f_shared + 127) / 128; c1.b_group_rows = 0;
        c1.b_tile_rows = 128; c1.mma_n = 256; c1.out = a.h_shared; c1.ldo = a.f_shared; c1.out_row0 = 0;
        c1.out_rows = a.T;
        c1.a_scale = b.sxs; c1.b_scale = q.s1s; c1.b_scale2 = q.s3s; c1.b_scale_stride = 0;
        c0.ksplit = c1.ksplit = 1;
        p.offsets = routed ? a.offsets : nullptr;
        p.mprefix = a.mprefix;
        p.E = a.E;
        p.dense_rows = shared ? a.T : 0;
        p.b_slot = GEMM_B_BYTES;
        p.stages = GEMM_STAGES;
        p.group_map = a.group_map;
        long long tiles = 0;
        const int bm = a.pair ? PAIR_BM : GEMM_BM;
        if (routed) tiles += ((long long)(a.max_rows + bm - 1) / bm + a.E) * c0.ntiles;
        if (shared) tiles += (long long)((a.T + bm - 1) / bm) * c1.ntiles;
        PairSwapMaps sw;
        if (a.pair && (rc = make_swap_maps(&sw, true, routed ? b.xq : nullptr, a.d, a.max_rows,
                                           shared ? b.xqs : nullptr, a.d, a.T, routed ? q.W1q : nullptr,
                                           routed ? q.W3q : nullptr, weight_groups(a) * a.f,
                                           shared ? q.W1sq : nullptr, shared ? q.W3sq : nullptr, a.f_shared)) !=
                          MOE_OK)
            return rc;
        rc = a.pair ? launch_gemm_pair<EPI_SWIGLU, true>(di, A0, B0, B0b, A1, B1, B1b, p, sw, tiles, s)
                    : launch_gemm<EPI_SWIGLU, true>(di, A0, B0, B0b, A1, B1, B1b, p, tiles, s);
        if (rc != MOE_OK) return rc;
    }
    if (ev_down && cudaEventRecord(ev_down, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (routed && (rc = run_quant_h(a.h, n_routed, a.max_rows, a.f, b.hq, b.sh, s)) != MOE_OK) return rc;
    if (shared && (rc = run_quant_h(a.h_shared, nullptr, a.T, a.f_shared, b.hqs, b.shs, s)) != MOE_OK) return rc;
    if (ev_gemm2 && cudaEventRecord(ev_gemm2, s) != cudaSuccess) return MOE_ERR_CUDA;
    // ---- GEMM2: y = s_h s2 (hq W2q^T)
    {
        CUtensorMap A0, B0, A1, B1;
        if (routed) {
            if ((rc = make_map_e4m3(&A0, b.hq, a.f, a.max_rows, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map_e4m3(&B0, q.W2q, a.f, weight_groups(a) * a.d, a.pair ? 128 : 256)) != MOE_OK) return rc;
        }
        if (shared) {
            if ((rc = make_map_e4m3(&A1, b.hqs, a.f_shared, a.T, GEMM_BM)) != MOE_OK) return rc;
            if ((rc = make_map_e4m3(&B1, q.W2sq, a.f_shared, a.d, a.pair ? 128 : 256)) != MOE_OK) return rc;
        }
        if (!routed) { A0 = A1; B0 = B1; }
        if (!shared) { A1 = A0; B1 = B0; }
        GemmParams p;
        memset(&p, 0, sizeof(p));
        GemmClass& c0 = p.cls[0];
        c0.K = a.f; c0.n_out = a.d; c0.ntiles = (a.d + 255) / 256; c0.b_group_rows = a.d; c0.b_tile_rows = 256;
        c0.mma_n = 256; c0.out = a.y_perm; c0.ldo = a.d; c0.out_row0 = 0; c0.out_rows = a.max_rows;
        c0.a_scale = b.sh; c0.b_scale = q.s2; c0.b_scale_stride = a.d;
        GemmClass& c1 = p.cls[1];
        c1.K = a.f_shared; c1.n_out = a.d; c1.ntiles = (a.d + 255) / 256; c1.b_group_rows = 0; c1.b_tile_rows = 256;
        c1.mma_n = 256; c1.out = a.y_shared; c1.ldo = a.d; c1.out_row0 = 0; c1.out_rows = a.T;
        c1.a_scale = b.shs; c1.b_scale = q.s2s; c1.b_scale_stride = 0;
        c0.ksplit = c1.ksplit = 1;
        p.offsets = routed ? a.offsets : nullptr;
        p.mprefix = a.mprefix;
        p.E = a.E;
        p.dense_rows = shared ? a.T : 0;
        p.b_slot = GEMM_B_BYTES;
        p.stages = GEMM_STAGES;
        p.group_map = a.group_map;
        long long tiles = 0;
        const int bm = a.pair ? PAIR_BM : GEMM_BM;
        if (routed) tiles += ((long long)(a.max_rows + bm - 1) / bm + a.E) * c0.ntiles;
        if (shared) tiles += (long long)((a.T + bm - 1) / bm) * c1.ntiles;
        PairSwapMaps sw;
        if (a.pair && (rc = make_swap_maps(&sw, true, routed ? b.hq : nullptr, a.f, a.max_rows,
                                           shared ? b.hqs : nullptr, a.f_shared, a.T, nullptr, nullptr, 0, nullptr,
                                           nullptr, 0)) != MOE_OK)
            return rc;
        rc = a.pair ? launch_gemm_pair<EPI_STORE, true>(di, A0, B0, B0, A1, B1, B1, p, sw, tiles, s)
                    : launch_gemm<EPI_STORE, true>(di, A0, B0, B0, A1, B1, B1, p, tiles, s);
        if (rc != MOE_OK) return rc;
    }
    return MOE_OK;
}

int run_combine(const moe_bf16* y_perm, const int32_t* dest, const float* w, const moe_bf16* y_shared, int T, int d,
                int k, moe_bf16* out, cudaStream_t s) {
    // longest row segment per warp that still leaves >= 8192 warps (or one 32-chunk segment)
    const int nvec = d / 8;
    int seg = 1;
    while (32 * seg * 2 <= nvec && (long long)T * ((nvec + 64 * seg - 1) / (64 * seg)) >= 8192) seg *= 2;
    const long long warps = (long long)T * ((nvec + 32 * seg - 1) / (32 * seg));
    combine_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(reinterpret_cast<const uint4*>(y_perm), dest, w,
                                                                reinterpret_cast<const uint4*>(y_shared), T, d, k,
                                                                seg, reinterpret_cast<uint4*>(out));
    return launch_status();
}

}  // namespace
}  // namespace moe

using namespace moe;

#define MOE_REQUIRE(cond, code) \
    do {                        \
        if (!(cond)) return (code); \
    } while (0)

extern "C" {

int64_t moe_capacity(int T, int E, int k, double capacity_factor, int cap_mode) {
    if (E <= 0) return -1;
    if (cap_mode == MOE_CAP_PER_TOKEN) return (int64_t)((double)T / (double)E * capacity_factor);
    if (cap_mode == MOE_CAP_PER_ASSIGNMENT) return (int64_t)((double)T * (double)k / (double)E * capacity_factor);
    return -1;
}

int moe_workspace_bytes(int T, int d, int E, int k, int f, int f_shared, size_t* bytes) {
    MOE_REQUIRE(bytes != nullptr, MOE_ERR_INVALID_ARG);
    int rc = check_shape(T, d, E, k, f);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(f_shared >= 0 && f_shared % 64 == 0, MOE_ERR_SHAPE);
    *bytes = layer_layout(T, d, E, k, f, f_shared).total;
    return MOE_OK;
}

int moe_workspace_layout(int T, int d, int E, int k, int f, int f_shared, size_t off[13]) {
    MOE_REQUIRE(off != nullptr, MOE_ERR_INVALID_ARG);
    int rc = check_shape(T, d, E, k, f);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(f_shared >= 0 && f_shared % 64 == 0, MOE_ERR_SHAPE);
    LayerLayout L = layer_layout(T, d, E, k, f, f_shared);
    for (int i = 0; i < 12; ++i) off[i] = L.off[i];
    off[12] = L.h_shared;
    return MOE_OK;
}

int moe_route(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const float* logits_in, int T, int d, int E,
              int k, float* logits_out, int32_t* idx, float* w, void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_REQUIRE(T >= 1 && k >= 1 && k <= MAX_TOPK && E >= k && E <= 1024 && (long long)T * k < (1ll << 31),
                MOE_ERR_SHAPE);
    MOE_REQUIRE(idx && w, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(idx) && aligned16(w) && aligned16(bias) && aligned16(logits_in) && aligned16(logits_out),
                MOE_ERR_ALIGN);
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!logits_in) {
        MOE_REQUIRE(x && Wg, MOE_ERR_INVALID_ARG);
        MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_SHAPE);
        MOE_REQUIRE(aligned16(x) && aligned16(Wg), MOE_ERR_ALIGN);
        const int ks = router_ksplit(T, d, E);
        const size_t own = logits_out ? 0 : align256((size_t)T * E * 4);
        const size_t need = own + (ks > 1 ? (size_t)ks * T * E * 4 : 0);
        MOE_REQUIRE(need == 0 || (ws && ws_bytes >= need), MOE_ERR_WORKSPACE);
        MOE_REQUIRE(aligned16(ws), MOE_ERR_ALIGN);
        float* dst = logits_out ? logits_out : static_cast<float*>(ws);
        float* part = ks > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + own) : nullptr;
        if ((rc = run_router_gemm(di, x, Wg, T, d, E, dst, part, ks, s)) != MOE_OK) return rc;
        return ks > 1 ? run_topk(part, ks, dst, bias, T, E, k, idx, w, s)
                      : run_topk(dst, 1, nullptr, bias, T, E, k, idx, w, s);
    }
    if (logits_out && logits_out != logits_in) {
        if (cudaMemcpyAsync(logits_out, logits_in, (size_t)T * E * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    return run_topk(logits_in, 1, nullptr, bias, T, E, k, idx, w, s);
}

int moe_permute(const moe_bf16* x, const int32_t* idx, int T, int d, int E, int k, int64_t capacity,
                int32_t* counts_raw, int32_t* counts, int32_t* offsets, int32_t* dest, int32_t* src_token,
                moe_bf16* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
    int rc = check_shape(T, d, E, k, 64);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(x && idx && counts_raw && counts && offsets && dest && src_token && x_perm && ws, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x) && aligned16(x_perm) && aligned16(idx) && aligned16(dest) && aligned16(ws),
                MOE_ERR_ALIGN);
    size_t o_blk, o_rank, o_mp;
    const size_t need = permute_scratch_bytes(T, E, k, &o_blk, &o_rank, &o_mp);
    MOE_REQUIRE(ws_bytes >= need, MOE_ERR_WORKSPACE);
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    char* base = static_cast<char*>(ws);
    return run_permute(di, x, idx, T, d, E, k, capacity < 0 ? -1 : (long long)capacity, counts_raw, counts, offsets,
                       dest, src_token, x_perm, reinterpret_cast<int32_t*>(base + o_blk),
                       reinterpret_cast<int32_t*>(base + o_rank), reinterpret_cast<int32_t*>(base + o_mp),
                       static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn(const moe_bf16* x_perm, const int32_t* offsets, int max_rows, int E, int d, int f,
                   const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2, moe_bf16* h, moe_bf16* y_perm,
                   void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_REQUIRE(max_rows >= 0 && E >= 1 && E <= 1024 && d >= 64 && d % 64 == 0 && f >= 64 && f % 64 == 0,
                MOE_ERR_SHAPE);
    MOE_REQUIRE(x_perm && offsets && W1 && W3 && W2 && h && y_perm && ws, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x_perm) && aligned16(W1) && aligned16(W3) && aligned16(W2) && aligned16(h) &&
                    aligned16(y_perm) && aligned16(ws),
                MOE_ERR_ALIGN);
    MOE_REQUIRE(ws_bytes >= (size_t)(E + 1) * 4, MOE_ERR_WORKSPACE);
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    if (max_rows == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* mprefix = static_cast<int32_t*>(ws);
    const bool pair = use_pair_tiles(max_rows, E);
    tile_prefix_kernel<<<1, 1024, 0, s>>>(offsets, E, max_rows, pair ? PAIR_BM : GEMM_BM, mprefix);
    if ((rc = launch_status()) != MOE_OK) return rc;
    FfnArgs a;
    memset(&a, 0, sizeof(a));
    a.x_perm = x_perm; a.offsets = offsets; a.mprefix = mprefix; a.max_rows = max_rows; a.E = E; a.d = d; a.f = f;
    a.W1 = W1; a.W3 = W3; a.W2 = W2; a.h = h; a.y_perm = y_perm;
    a.f_shared = 0;
    a.pair = pair;
    return run_expert_ffn(di, a, s);
}

int moe_combine(const moe_bf16* y_perm, const int32_t* dest, const float* w, const moe_bf16* y_shared, int T, int d,
                int k, moe_bf16* out, moe_stream_t stream) {
    MOE_REQUIRE(T >= 1 && d >= 64 && d % 64 == 0 && k >= 1 && k <= MAX_TOPK, MOE_ERR_SHAPE);
    MOE_REQUIRE(y_perm && dest && w && out, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(y_perm) && aligned16(y_shared) && aligned16(out), MOE_ERR_ALIGN);
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    return run_combine(y_perm, dest, w, y_shared, T, d, k, out, static_cast<cudaStream_t>(stream));
}

int moe_layer_forward(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_bf16* W1, const moe_bf16* W3,
                      const moe_bf16* W2, const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s, int f_shared,
                      int T, int d, int E, int k, int f, double capacity_factor, int cap_mode, moe_bf16* out, void* ws,
                      size_t ws_bytes, moe_stream_t stream) {
    return moe_layer_forward_ex(x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, capacity_factor,
                                cap_mode, out, ws, ws_bytes, stream, nullptr);
}

}  // extern "C"

namespace moe {
namespace {

enum { LAYER_ROUTE = 1, LAYER_COUNT = 2, LAYER_FINISH = 4, LAYER_PERMUTE = 8, LAYER_INDICES = 16 };

// The layer in phases over one workspace:
//   LAYER_ROUTE   router GEMM + top-k                 (needs x, Wg, bias)
//   LAYER_COUNT   histogram only: counts_raw          (no capacity)
//   LAYER_PERMUTE histogram, capacity (with fill_base), permutation; stops there
//   LAYER_FINISH  histogram, capacity (with fill_base), permutation, experts, combine
// Routed expert weights served from the expert cache (moe_layer_forward_cached[_w8]).  cp lists
// the per-expert arrays to copy (device-usable source addresses, slot arrays); the GEMMs then
// read the slots (bf16: W1/W3/W2 arguments of layer_phases; fp8: its W8Weights) through slot_of.
struct CacheArgs {
    CacheCopy cp;
    int S;
    void* state;
};

int layer_phases(int phases, const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_bf16* W1,
                 const moe_bf16* W3, const moe_bf16* W2, const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s,
                 int f_shared, int T, int d, int E, int k, int f, long long C, const int32_t* fill_base,
                 moe_bf16* out, void* ws, size_t ws_bytes, cudaStream_t s, const moe_stage_events* events,
                 const W8Weights* w8 = nullptr, const CacheArgs* cache = nullptr, bool act8 = false) {
    int rc = check_shape(T, d, E, k, f);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(f_shared >= 0 && f_shared % 64 == 0, MOE_ERR_SHAPE);
    MOE_REQUIRE(x && ws, MOE_ERR_INVALID_ARG);
    if (phases & LAYER_ROUTE) MOE_REQUIRE(Wg, MOE_ERR_INVALID_ARG);
    const bool shared = f_shared > 0;
    if ((phases & LAYER_FINISH) && !w8) {
        MOE_REQUIRE(W1 && W3 && W2 && out, MOE_ERR_INVALID_ARG);
        MOE_REQUIRE(!shared || (W1s && W3s && W2s), MOE_ERR_INVALID_ARG);
    }
    if ((phases & LAYER_FINISH) && w8) {
        MOE_REQUIRE(w8->W1q && w8->W3q && w8->W2q && w8->s1 && w8->s3 && w8->s2 && out, MOE_ERR_INVALID_ARG);
        MOE_REQUIRE(!shared || (w8->W1sq && w8->W3sq && w8->W2sq && w8->s1s && w8->s3s && w8->s2s),
                    MOE_ERR_INVALID_ARG);
        MOE_REQUIRE(aligned16(w8->W1q) && aligned16(w8->W3q) && aligned16(w8->W2q) && aligned16(w8->W1sq) &&
                        aligned16(w8->W3sq) && aligned16(w8->W2sq) && aligned16(w8->s1) && aligned16(w8->s3) &&
                        aligned16(w8->s2) && aligned16(w8->s1s) && aligned16(w8->s3s) && aligned16(w8->s2s),
                    MOE_ERR_ALIGN);
    }
    MOE_REQUIRE(aligned16(x) && aligned16(Wg) && aligned16(bias) && aligned16(W1) && aligned16(W3) && aligned16(W2) &&
                    aligned16(W1s) && aligned16(W3s) && aligned16(W2s) && aligned16(out) && aligned16(ws) &&
                    aligned16(fill_base),
                MOE_ERR_ALIGN);
    const LayerLayout L = layer_layout(T, d, E, k, f, f_shared);
    MOE_REQUIRE(ws_bytes >= L.total, MOE_ERR_WORKSPACE);
    const A8Layout A8 = a8_layout(L.total, T, d, k, f, f_shared);
    if (act8) MOE_REQUIRE(ws_bytes >= A8.total, MOE_ERR_WORKSPACE);
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    char* base = static_cast<char*>(ws);
    float* logits = reinterpret_cast<float*>(base + L.off[0]);
    int32_t* idx = reinterpret_cast<int32_t*>(base + L.off[1]);
    float* w = reinterpret_cast<float*>(base + L.off[2]);
    int32_t* counts_raw = reinterpret_cast<int32_t*>(base + L.off[3]);
    int32_t* counts = reinterpret_cast<int32_t*>(base + L.off[4]);
    int32_t* offsets = reinterpret_cast<int32_t*>(base + L.off[5]);
    int32_t* dest = reinterpret_cast<int32_t*>(base + L.off[6]);
    int32_t* src = reinterpret_cast<int32_t*>(base + L.off[7]);
    moe_bf16* x_perm = reinterpret_cast<moe_bf16*>(base + L.off[8]);
    moe_bf16* h = reinterpret_cast<moe_bf16*>(base + L.off[9]);
    moe_bf16* y_perm = reinterpret_cast<moe_bf16*>(base + L.off[10]);
    moe_bf16* y_shared = shared ? reinterpret_cast<moe_bf16*>(base + L.off[11]) : nullptr;
    moe_bf16* h_shared = shared ? reinterpret_cast<moe_bf16*>(base + L.h_shared) : nullptr;
    int32_t* blk_cnt = reinterpret_cast<int32_t*>(base + L.blk_cnt);
    int32_t* rank_local = reinterpret_cast<int32_t*>(base + L.rank_local);
    int32_t* mprefix = reinterpret_cast<int32_t*>(base + L.mprefix);

    moe_stage_events ev;
    memset(&ev, 0, sizeof(ev));
    if (events) ev = *events;
    auto mark = [&](void* e) { return e == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(e), s) == cudaSuccess; };

    if (phases & LAYER_ROUTE) {
        if (!mark(ev.route)) return MOE_ERR_CUDA;
        const int ks = router_ksplit(T, d, E);
        float* part = reinterpret_cast<float*>(base + L.router_part);
        if ((rc = run_router_gemm(di, x, Wg, T, d, E, logits, part, ks, s)) != MOE_OK) return rc;
        if (!mark(ev.topk)) return MOE_ERR_CUDA;
        rc = ks > 1 ? run_topk(part, ks, logits, bias, T, E, k, idx, w, s)
                    : run_topk(logits, 1, nullptr, bias, T, E, k, idx, w, s);
        if (rc != MOE_OK) return rc;
    }
    // weight-only fp8: 1-SM tiles (its own kernel); bf16 and fp8 x fp8: 2-SM tiles for big experts
    const bool pair = (!w8 || act8) && use_pair_tiles((long long)T * k, E);
    if (phases & LAYER_COUNT) {
        if ((rc = run_permute(di, x, idx, T, d, E, k, -1, counts_raw, counts, offsets, dest, src, x_perm, blk_cnt,
                              rank_local, mprefix, s, GEMM_BM, nullptr, true)) != MOE_OK)
            return rc;
    }
    if (phases & (LAYER_PERMUTE | LAYER_INDICES))   // LAYER_INDICES: dest / src_token only, no x_perm
        return run_permute(di, x, idx, T, d, E, k, C, counts_raw, counts, offsets, dest, src, x_perm, blk_cnt,
                           rank_local, mprefix, s, GEMM_BM, fill_base, false, !(phases & LAYER_INDICES));
    if (!(phases & LAYER_FINISH)) return MOE_OK;
    if (!mark(ev.permute)) return MOE_ERR_CUDA;
    // fp8 activations: each x row is quantised once and written to its rows by dest: no x_perm
    if ((rc = run_permute(di, x, idx, T, d, E, k, C, counts_raw, counts, offsets, dest, src, x_perm, blk_cnt,
                          rank_local, mprefix, s, pair ? PAIR_BM : GEMM_BM, fill_base, false, !(w8 && act8))) != MOE_OK)
        return rc;
    CacheView cv{};
    int32_t* mp_hit = reinterpret_cast<int32_t*>(base + L.mp_hit);
    int32_t* mp_miss = reinterpret_cast<int32_t*>(base + L.mp_miss);
    if (cache) {
        // plan on the layer's stream; the copy of the missed experts on the copy stream, which
        // forks after the plan and joins before the misses' GEMMs
        if ((rc = copy_stream(di)) != MOE_OK) return rc;
        if (!mark(ev.cache)) return MOE_ERR_CUDA;
        cv = cache_view(cache->state, E, cache->S);
        cache_plan_kernel<<<1, CACHE_MAX, 0, s>>>(counts, E, cache->S, cv, pair ? PAIR_BM : GEMM_BM, mp_hit, mp_miss);
        if ((rc = launch_status()) != MOE_OK) return rc;
        if (cudaEventRecord(di->copy_fork, s) != cudaSuccess ||
            cudaStreamWaitEvent(di->copy_stream, di->copy_fork, 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (ev.copy_start && cudaEventRecord(static_cast<cudaEvent_t>(ev.copy_start), di->copy_stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        cache_load_kernel<<<2 * di->sms, CACHE_LOAD_THREADS, 0, di->copy_stream>>>(cv.ctr, cv.load_expert,
                                                                                   cv.load_slot, cache->cp);
        if ((rc = launch_status()) != MOE_OK) return rc;
        if (ev.copy_end && cudaEventRecord(static_cast<cudaEvent_t>(ev.copy_end), di->copy_stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaEventRecord(di->copy_join, di->copy_stream) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (!mark(ev.gate_up)) return MOE_ERR_CUDA;
    FfnArgs a;
    memset(&a, 0, sizeof(a));
    a.x_perm = x_perm; a.offsets = offsets; a.mprefix = mprefix; a.max_rows = T * k; a.E = E; a.d = d; a.f = f;
    a.W1 = W1; a.W3 = W3; a.W2 = W2; a.h = h; a.y_perm = y_perm;
    if (cache) {     // W1/W3/W2 (or w8) already point at the slots; first the resident experts
        a.group_map = cv.slot_of;
        a.w_groups = cache->S;
        a.mprefix = mp_hit;
    }
    a.x = x; a.T = T; a.f_shared = f_shared; a.W1s = W1s; a.W3s = W3s; a.W2s = W2s;
    a.h_shared = h_shared; a.y_shared = y_shared;
    a.pair = pair;
    if (w8 && act8) {
        A8Bufs b;
        b.xq = reinterpret_cast<uint8_t*>(base + A8.xq);
        b.hq = reinterpret_cast<uint8_t*>(base + A8.hq);
        b.xqs = shared ? reinterpret_cast<uint8_t*>(base + A8.xqs) : nullptr;
        b.hqs = shared ? reinterpret_cast<uint8_t*>(base + A8.hqs) : nullptr;
        b.sx = reinterpret_cast<float*>(base + A8.sx);
        b.sh = reinterpret_cast<float*>(base + A8.sh);
        b.sxs = shared ? reinterpret_cast<float*>(base + A8.sxs) : nullptr;
        b.shs = shared ? reinterpret_cast<float*>(base + A8.shs) : nullptr;
        b.dest = dest;
        b.src_token = src;
        b.k = k;
        rc = run_expert_ffn_a8(di, a, *w8, b, s, static_cast<cudaEvent_t>(ev.down), static_cast<cudaEvent_t>(ev.gemm1),
                               static_cast<cudaEvent_t>(ev.gemm2));
    } else {
        rc = w8 ? run_expert_ffn_w8(di, a, *w8, s, static_cast<cudaEvent_t>(ev.down))
                : run_expert_ffn(di, a, s, static_cast<cudaEvent_t>(ev.down));
        if (rc == MOE_OK && cache) {
            // then the experts this batch loaded, once their copy is done (routed groups only)
            if (cudaStreamWaitEvent(s, di->copy_join, 0) != cudaSuccess) return MOE_ERR_CUDA;
            FfnArgs m = a;
            m.mprefix = mp_miss;
            m.f_shared = 0;
            m.h_shared = m.y_shared = nullptr;
            m.W1s = m.W3s = m.W2s = nullptr;
            W8Weights qm;
            if (w8) {
                qm = *w8;
                qm.W1sq = qm.W3sq = qm.W2sq = nullptr;
                qm.s1s = qm.s3s = qm.s2s = nullptr;
            }
            rc = w8 ? run_expert_ffn_w8(di, m, qm, s, nullptr) : run_expert_ffn(di, m, s);
        }
    }
    if (rc != MOE_OK) return rc;
    if (!mark(ev.combine)) return MOE_ERR_CUDA;
    if ((rc = run_combine(y_perm, dest, w, y_shared, T, d, k, out, s)) != MOE_OK) return rc;
    return mark(ev.end) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_layer_forward_ex(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_bf16* W1,
                         const moe_bf16* W3, const moe_bf16* W2, const moe_bf16* W1s, const moe_bf16* W3s,
                         const moe_bf16* W2s, int f_shared, int T, int d, int E, int k, int f, double capacity_factor,
                         int cap_mode, moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                         const moe_stage_events* events) {
    MOE_REQUIRE(cap_mode >= MOE_CAP_NONE && cap_mode <= MOE_CAP_PER_ASSIGNMENT, MOE_ERR_INVALID_ARG);
    const long long C = moe_capacity(T, E, k, capacity_factor, cap_mode);
    return layer_phases(LAYER_ROUTE | LAYER_FINISH, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f, C,
                        nullptr, out, ws, ws_bytes, static_cast<cudaStream_t>(stream), events);
}

int moe_cache_state_bytes(int E, int S, size_t* bytes) {
    MOE_REQUIRE(bytes, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(S >= 1 && S <= E && E <= moe::CACHE_MAX, MOE_ERR_SHAPE);
    size_t off[6];
    *bytes = moe::cache_layout(E, S, off);
    return MOE_OK;
}

int moe_cache_layout(int E, int S, size_t off[6]) {
    MOE_REQUIRE(off, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(S >= 1 && S <= E && E <= moe::CACHE_MAX, MOE_ERR_SHAPE);
    moe::cache_layout(E, S, off);
    return MOE_OK;
}

int moe_cache_reset(void* cache_state, int E, int S, moe_stream_t stream) {
    using namespace moe;
    MOE_REQUIRE(cache_state, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(cache_state), MOE_ERR_ALIGN);
    MOE_REQUIRE(S >= 1 && S <= E && E <= CACHE_MAX, MOE_ERR_SHAPE);
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cache_reset_kernel<<<1, CACHE_MAX, 0, static_cast<cudaStream_t>(stream)>>>(cache_view(cache_state, E, S), E, S);
    return launch_status();
}

// Address the device uses for a cache source: page-locked host memory (mapped) or device memory.
static int cache_source(const void* p, const uint4** dev) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_INVALID_ARG;
    }
    if (at.type == cudaMemoryTypeHost && at.devicePointer) *dev = static_cast<const uint4*>(at.devicePointer);
    else if (at.type == cudaMemoryTypeDevice) *dev = static_cast<const uint4*>(p);
    else return MOE_ERR_INVALID_ARG;   // pageable host memory (or unknown)
    return MOE_OK;
}

int moe_layer_forward_cached(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_bf16* W1_src,
                             const moe_bf16* W3_src, const moe_bf16* W2_src, moe_bf16* W1_slots, moe_bf16* W3_slots,
                             moe_bf16* W2_slots, int S, void* cache_state, const moe_bf16* W1s, const moe_bf16* W3s,
                             const moe_bf16* W2s, int f_shared, int T, int d, int E, int k, int f,
                             double capacity_factor, int cap_mode, moe_bf16* out, void* ws, size_t ws_bytes,
                             moe_stream_t stream, const moe_stage_events* events) {
    using namespace moe;
    MOE_REQUIRE(cap_mode >= MOE_CAP_NONE && cap_mode <= MOE_CAP_PER_ASSIGNMENT, MOE_ERR_INVALID_ARG);
    int rc = check_shape(T, d, E, k, f);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(S >= 1 && S <= E && (long long)S >= std::min<long long>(E, (long long)T * k), MOE_ERR_SHAPE);
    MOE_REQUIRE(W1_src && W3_src && W2_src && W1_slots && W3_slots && W2_slots && cache_state, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(W1_src) && aligned16(W3_src) && aligned16(W2_src) && aligned16(W1_slots) &&
                    aligned16(W3_slots) && aligned16(W2_slots) && aligned16(cache_state),
                MOE_ERR_ALIGN);
    CacheArgs ca;
    memset(&ca, 0, sizeof(ca));
    const void* srcs[3] = {W1_src, W3_src, W2_src};
    void* dsts[3] = {W1_slots, W3_slots, W2_slots};
    for (int i = 0; i < 3; ++i) {
        if ((rc = cache_source(srcs[i], &ca.cp.src[i])) != MOE_OK) return rc;
        ca.cp.dst[i] = static_cast<uint4*>(dsts[i]);
        ca.cp.per[i] = (long long)f * d / 8;
    }
    ca.cp.n = 3;
    ca.S = S;
    ca.state = cache_state;
    const long long C = moe_capacity(T, E, k, capacity_factor, cap_mode);
    return layer_phases(LAYER_ROUTE | LAYER_FINISH, x, Wg, bias, W1_slots, W3_slots, W2_slots, W1s, W3s, W2s,
                        f_shared, T, d, E, k, f, C, nullptr, out, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                        events, nullptr, &ca);
}

int moe_layer_forward_cached_w8(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_w8_experts* src,
                                const moe_w8_slots* slots, int S, void* cache_state, const moe_w8_experts* shared,
                                int f_shared, int T, int d, int E, int k, int f, double capacity_factor, int cap_mode,
                                moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                                const moe_stage_events* events) {
    using namespace moe;
    MOE_REQUIRE(cap_mode >= MOE_CAP_NONE && cap_mode <= MOE_CAP_PER_ASSIGNMENT, MOE_ERR_INVALID_ARG);
    int rc = check_shape(T, d, E, k, f);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(S >= 1 && S <= E && (long long)S >= std::min<long long>(E, (long long)T * k), MOE_ERR_SHAPE);
    MOE_REQUIRE(src && slots && cache_state && (f_shared == 0 || shared), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(src->W1q && src->W3q && src->W2q && src->s1 && src->s3 && src->s2, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(slots->W1q && slots->W3q && slots->W2q && slots->s1 && slots->s3 && slots->s2, MOE_ERR_INVALID_ARG);
    const void* sp[6] = {src->W1q, src->W3q, src->W2q, src->s1, src->s3, src->s2};
    void* dp[6] = {slots->W1q, slots->W3q, slots->W2q, slots->s1, slots->s3, slots->s2};
    for (int i = 0; i < 6; ++i) MOE_REQUIRE(aligned16(sp[i]) && aligned16(dp[i]), MOE_ERR_ALIGN);
    MOE_REQUIRE(aligned16(cache_state), MOE_ERR_ALIGN);
    CacheArgs ca;
    memset(&ca, 0, sizeof(ca));
    const long long per[6] = {(long long)f * d / 16, (long long)f * d / 16, (long long)d * f / 16,
                              (long long)f * 4 / 16, (long long)f * 4 / 16, (long long)d * 4 / 16};
    for (int i = 0; i < 6; ++i) {
        if ((rc = cache_source(sp[i], &ca.cp.src[i])) != MOE_OK) return rc;
        ca.cp.dst[i] = static_cast<uint4*>(dp[i]);
        ca.cp.per[i] = per[i];
    }
    ca.cp.n = 6;
    ca.S = S;
    ca.state = cache_state;
    W8Weights q = {slots->W1q, slots->W3q, slots->W2q,
                   shared ? shared->W1q : nullptr, shared ? shared->W3q : nullptr, shared ? shared->W2q : nullptr,
                   slots->s1, slots->s3, slots->s2,
                   shared ? shared->s1 : nullptr, shared ? shared->s3 : nullptr, shared ? shared->s2 : nullptr};
    const long long C = moe_capacity(T, E, k, capacity_factor, cap_mode);
    return layer_phases(LAYER_ROUTE | LAYER_FINISH, x, Wg, bias, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        f_shared, T, d, E, k, f, C, nullptr, out, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                        events, &q, &ca);
}

int moe_workspace_bytes_a8(int T, int d, int E, int k, int f, int f_shared, size_t* bytes) {
    using namespace moe;
    MOE_REQUIRE(bytes, MOE_ERR_INVALID_ARG);
    int rc = check_shape(T, d, E, k, f);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(f_shared >= 0 && f_shared % 64 == 0, MOE_ERR_SHAPE);
    *bytes = a8_layout(layer_layout(T, d, E, k, f, f_shared).total, T, d, k, f, f_shared).total;
    return MOE_OK;
}

int moe_layer_forward_w8a8(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const uint8_t* W1q,
                           const float* s1, const uint8_t* W3q, const float* s3, const uint8_t* W2q, const float* s2,
                           const uint8_t* W1sq, const float* s1s, const uint8_t* W3sq, const float* s3s,
                           const uint8_t* W2sq, const float* s2s, int f_shared, int T, int d, int E, int k, int f,
                           double capacity_factor, int cap_mode, moe_bf16* out, void* ws, size_t ws_bytes,
                           moe_stream_t stream, const moe_stage_events* events) {
    MOE_REQUIRE(cap_mode >= MOE_CAP_NONE && cap_mode <= MOE_CAP_PER_ASSIGNMENT, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(d % 128 == 0 && f % 128 == 0 && f_shared % 128 == 0, MOE_ERR_SHAPE);   // 128-byte fp8 K rows
    const long long C = moe_capacity(T, E, k, capacity_factor, cap_mode);
    moe::W8Weights q = {W1q, W3q, W2q, W1sq, W3sq, W2sq, s1, s3, s2, s1s, s3s, s2s};
    return moe::layer_phases(moe::LAYER_ROUTE | moe::LAYER_FINISH, x, Wg, bias, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, f_shared, T, d, E, k, f, C, nullptr, out, ws, ws_bytes,
                             static_cast<cudaStream_t>(stream), events, &q, nullptr, true);
}

int moe_layer_forward_w8(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const uint8_t* W1q,
                         const float* s1, const uint8_t* W3q, const float* s3, const uint8_t* W2q, const float* s2,
                         const uint8_t* W1sq, const float* s1s, const uint8_t* W3sq, const float* s3s,
                         const uint8_t* W2sq, const float* s2s, int f_shared, int T, int d, int E, int k, int f,
                         double capacity_factor, int cap_mode, moe_bf16* out, void* ws, size_t ws_bytes,
                         moe_stream_t stream, const moe_stage_events* events) {
    MOE_REQUIRE(cap_mode >= MOE_CAP_NONE && cap_mode <= MOE_CAP_PER_ASSIGNMENT, MOE_ERR_INVALID_ARG);
    const long long C = moe_capacity(T, E, k, capacity_factor, cap_mode);
    W8Weights q = {W1q, W3q, W2q, W1sq, W3sq, W2sq, s1, s3, s2, s1s, s3s, s2s};
    return layer_phases(LAYER_ROUTE | LAYER_FINISH, x, Wg, bias, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        f_shared, T, d, E, k, f, C, nullptr, out, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                        events, &q);
}

int moe_layer_route_count(const moe_bf16* x, const moe_bf16* Wg, const float* bias, int f_shared, int T, int d, int E,
                          int k, int f, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return layer_phases(LAYER_ROUTE | LAYER_COUNT, x, Wg, bias, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        f_shared, T, d, E, k, f, -1, nullptr, nullptr, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                        nullptr);
}

int moe_fill_base(const int32_t* all_counts, int G, int rank, int E, int32_t* fill_base, moe_stream_t stream) {
    MOE_REQUIRE(G >= 1 && rank >= 0 && rank < G && E >= 1 && E <= 1024, MOE_ERR_SHAPE);
    MOE_REQUIRE(all_counts && fill_base, MOE_ERR_INVALID_ARG);
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    fill_base_kernel<<<(E + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(all_counts, G, rank, E,
                                                                                    fill_base);
    return launch_status();
}

int moe_layer_finish(const moe_bf16* x, const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2,
                     const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s, int f_shared, int T, int d, int E,
                     int k, int f, int64_t capacity, const int32_t* fill_base, moe_bf16* out, void* ws,
                     size_t ws_bytes, moe_stream_t stream) {
    return layer_phases(LAYER_FINISH, x, nullptr, nullptr, W1, W3, W2, W1s, W3s, W2s, f_shared, T, d, E, k, f,
                        capacity < 0 ? -1 : (long long)capacity, fill_base, out, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream), nullptr);
}

int moe_layer_permute(const moe_bf16* x, int f_shared, int T, int d, int E, int k, int f, int64_t capacity,
                      const int32_t* fill_base, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return layer_phases(LAYER_PERMUTE, x, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        f_shared, T, d, E, k, f, capacity < 0 ? -1 : (long long)capacity, fill_base, nullptr, ws,
                        ws_bytes, static_cast<cudaStream_t>(stream), nullptr);
}

int moe_layer_permute_indices(const moe_bf16* x, int f_shared, int T, int d, int E, int k, int f, int64_t capacity,
                              const int32_t* fill_base, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return layer_phases(LAYER_INDICES, x, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        f_shared, T, d, E, k, f, capacity < 0 ? -1 : (long long)capacity, fill_base, nullptr, ws,
                        ws_bytes, static_cast<cudaStream_t>(stream), nullptr);
}

// ------------------------------------------------------------------ expert parallelism

namespace {

int ep_check(int R, int rank, int E, int d) {
    MOE_REQUIRE(R >= 1 && R <= moe::EP_MAX_RANKS && rank >= 0 && rank < R, MOE_ERR_SHAPE);
    MOE_REQUIRE(E >= 1 && E <= moe::EP_MAX_EXPERTS && E % R == 0, MOE_ERR_SHAPE);
    MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_SHAPE);
    return MOE_OK;
}

size_t ep_bytes(int R, int E) {
    size_t off[9];
    return moe::ep_layout_bytes(R, E, off);
}

int ep_put(const void* src, const int32_t* table, moe_bf16* const* dests, int R, int E, int d, cudaStream_t s) {
    using namespace moe;
    EpDests dst;
    memset(&dst, 0, sizeof(dst));
    for (int q = 0; q < R; ++q) {
        MOE_REQUIRE(dests[q] && aligned16(dests[q]), MOE_ERR_INVALID_ARG);
        dst.base[q] = reinterpret_cast<char*>(dests[q]);
    }
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    const int bx = std::max(1, std::min(8, (2 * di->sms + E - 1) / E));
    ep_put_rows_kernel<<<dim3(bx, E), 256, 0, s>>>(table, E, E / R, static_cast<const uint4*>(src), dst,
                                                    (long long)d / 8);
    return launch_status();
}

}  // namespace

int moe_ep_workspace_bytes(int R, int E, size_t* bytes) {
    MOE_REQUIRE(bytes, MOE_ERR_INVALID_ARG);
    int rc = ep_check(R, 0, E, 64);
    if (rc != MOE_OK) return rc;
    *bytes = ep_bytes(R, E);
    return MOE_OK;
}

int moe_ep_splits_offset(int R, int E, size_t* offset) {
    MOE_REQUIRE(offset, MOE_ERR_INVALID_ARG);
    int rc = ep_check(R, 0, E, 64);
    if (rc != MOE_OK) return rc;
    size_t off[9];
    moe::ep_layout_bytes(R, E, off);
    *offset = off[8];
    return MOE_OK;
}

// ---- peer buffers: CUDA IPC handles of device allocations

namespace {

using cuMemGetAddressRange_t = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

cuMemGetAddressRange_t address_range_fn() {
    static cuMemGetAddressRange_t fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<cuMemGetAddressRange_t>(p);
    });
    return fn;
}

struct IpcBlob {                 // layout of the MOE_IPC_HANDLE_BYTES a handle occupies
    cudaIpcMemHandle_t mem;      // handle of the allocation that holds the pointer
    uint64_t offset;             // the pointer's offset from the allocation's base
    uint64_t magic;
};
static_assert(sizeof(IpcBlob) <= MOE_IPC_HANDLE_BYTES, "IPC handle blob");
constexpr uint64_t kIpcMagic = 0x6d6f652d69706331ull;

}  // namespace

int moe_ipc_export(const void* ptr, void* handle) {
    MOE_REQUIRE(ptr && handle, MOE_ERR_INVALID_ARG);
    cuMemGetAddressRange_t range = address_range_fn();
    if (!range) return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return MOE_ERR_INVALID_ARG;
    IpcBlob b;
    memset(&b, 0, sizeof(b));
    if (cudaIpcGetMemHandle(&b.mem, reinterpret_cast<void*>(base)) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    b.offset = reinterpret_cast<uint64_t>(ptr) - static_cast<uint64_t>(base);
    b.magic = kIpcMagic;
    memset(handle, 0, MOE_IPC_HANDLE_BYTES);
    memcpy(handle, &b, sizeof(b));
    return MOE_OK;
}

int moe_ipc_import(const void* handle, void** ptr) {
    MOE_REQUIRE(handle && ptr, MOE_ERR_INVALID_ARG);
    IpcBlob b;
    memcpy(&b, handle, sizeof(b));
    MOE_REQUIRE(b.magic == kIpcMagic, MOE_ERR_INVALID_ARG);
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, b.mem, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    *ptr = static_cast<char*>(base) + b.offset;
    return MOE_OK;
}

int moe_ipc_close(void* ptr, const void* handle) {
    MOE_REQUIRE(ptr && handle, MOE_ERR_INVALID_ARG);
    IpcBlob b;
    memcpy(&b, handle, sizeof(b));
    MOE_REQUIRE(b.magic == kIpcMagic, MOE_ERR_INVALID_ARG);
    if (cudaIpcCloseMemHandle(static_cast<char*>(ptr) - b.offset) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

int moe_ep_plan(const int32_t* all_counts_raw, int R, int rank, int E, int64_t capacity, int max_recv_rows,
                void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int rc = ep_check(R, rank, E, 64);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(max_recv_rows >= 0, MOE_ERR_SHAPE);
    MOE_REQUIRE(all_counts_raw && ep_ws, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(ep_ws), MOE_ERR_ALIGN);
    MOE_REQUIRE(ep_ws_bytes >= ep_bytes(R, E), MOE_ERR_WORKSPACE);
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    const bool pair = use_pair_tiles(max_recv_rows, E / R);
    ep_plan_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
        all_counts_raw, R, E, rank, capacity < 0 ? -1 : (long long)capacity, pair ? PAIR_BM : GEMM_BM,
        ep_view(ep_ws, R, E));
    return launch_status();
}

int moe_ep_dispatch(const moe_bf16* x_perm, int R, int rank, int E, int d, moe_bf16* const* recv_bufs,
                    const void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int rc = ep_check(R, rank, E, d);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(x_perm && recv_bufs && ep_ws, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x_perm) && aligned16(ep_ws), MOE_ERR_ALIGN);
    MOE_REQUIRE(ep_ws_bytes >= ep_bytes(R, E), MOE_ERR_WORKSPACE);
    const EpView v = ep_view(const_cast<void*>(ep_ws), R, E);
    return ep_put(x_perm, v.send, recv_bufs, R, E, d, static_cast<cudaStream_t>(stream));
}

int moe_ep_expert_ffn(const moe_bf16* recv_x, int max_recv_rows, int source_major, int R, int rank, int E, int d,
                      int f, const moe_bf16* W1_local, const moe_bf16* W3_local, const moe_bf16* W2_local, moe_bf16* h,
                      moe_bf16* y_recv, const moe_bf16* x, int T, const moe_bf16* W1s, const moe_bf16* W3s,
                      const moe_bf16* W2s, int f_shared, moe_bf16* h_shared, moe_bf16* y_shared, const void* ep_ws,
                      size_t ep_ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int rc = ep_check(R, rank, E, d);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(max_recv_rows >= 0 && f >= 64 && f % 64 == 0 && f_shared >= 0 && f_shared % 64 == 0, MOE_ERR_SHAPE);
    const bool shared = f_shared > 0;
    MOE_REQUIRE(ep_ws && (max_recv_rows == 0 || (recv_x && W1_local && W3_local && W2_local && h && y_recv)),
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!shared || (x && T >= 1 && W1s && W3s && W2s && h_shared && y_shared), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(recv_x) && aligned16(W1_local) && aligned16(W3_local) && aligned16(W2_local) &&
                    aligned16(h) && aligned16(y_recv) && aligned16(x) && aligned16(W1s) && aligned16(W3s) &&
                    aligned16(W2s) && aligned16(h_shared) && aligned16(y_shared) && aligned16(ep_ws),
                MOE_ERR_ALIGN);
    MOE_REQUIRE(ep_ws_bytes >= ep_bytes(R, E), MOE_ERR_WORKSPACE);
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    const EpView v = ep_view(const_cast<void*>(ep_ws), R, E);
    const int El = E / R;
    FfnArgs a;
    memset(&a, 0, sizeof(a));
    a.x_perm = recv_x;
    a.max_rows = max_recv_rows;
    if (source_major) {            // one segment per (source rank, local expert)
        a.offsets = v.seg_off;
        a.mprefix = v.seg_tiles;
        a.E = E;
        a.group_map = v.group_map;
        a.w_groups = El;
    } else {                       // expert-major: one group per local expert
        a.offsets = v.exp_off;
        a.mprefix = v.exp_tiles;
        a.E = El;
    }
    if (max_recv_rows == 0) a.offsets = nullptr;
    a.d = d;
    a.f = f;
    a.W1 = W1_local; a.W3 = W3_local; a.W2 = W2_local;
    a.h = h; a.y_perm = y_recv;
    a.x = x; a.T = T; a.f_shared = f_shared; a.W1s = W1s; a.W3s = W3s; a.W2s = W2s;
    a.h_shared = h_shared; a.y_shared = y_shared;
    a.pair = use_pair_tiles(max_recv_rows, El);
    if (max_recv_rows == 0 && !shared) return MOE_OK;
    return run_expert_ffn(di, a, static_cast<cudaStream_t>(stream));
}

int moe_ep_return(const moe_bf16* y_recv, int R, int rank, int E, int d, moe_bf16* const* y_perm_bufs,
                  const void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int rc = ep_check(R, rank, E, d);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(y_recv && y_perm_bufs && ep_ws, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(y_recv) && aligned16(ep_ws), MOE_ERR_ALIGN);
    MOE_REQUIRE(ep_ws_bytes >= ep_bytes(R, E), MOE_ERR_WORKSPACE);
    const EpView v = ep_view(const_cast<void*>(ep_ws), R, E);
    return ep_put(y_recv, v.back, y_perm_bufs, R, E, d, static_cast<cudaStream_t>(stream));
}

int moe_ep_dispatch_gather(const moe_bf16* x, const int32_t* src_token, int R, int rank, int E, int d,
                           moe_bf16* const* recv_bufs, const void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int rc = ep_check(R, rank, E, d);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(x && src_token && recv_bufs && ep_ws, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x) && aligned16(ep_ws), MOE_ERR_ALIGN);
    MOE_REQUIRE(ep_ws_bytes >= ep_bytes(R, E), MOE_ERR_WORKSPACE);
    EpDests dst;
    memset(&dst, 0, sizeof(dst));
    for (int q = 0; q < R; ++q) {
        MOE_REQUIRE(recv_bufs[q] && aligned16(recv_bufs[q]), MOE_ERR_INVALID_ARG);
        dst.base[q] = reinterpret_cast<char*>(recv_bufs[q]);
    }
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    const EpView v = ep_view(const_cast<void*>(ep_ws), R, E);
    const int bx = std::max(1, std::min(16, (4 * di->sms + E - 1) / E));
    ep_gather_put_kernel<<<dim3(bx, E), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        v.send, E, E / R, reinterpret_cast<const uint4*>(x), src_token, dst, d / 8);
    return launch_status();
}

int moe_ep_expert_ffn_return(const moe_bf16* recv_x, int max_recv_rows, int R, int rank, int E, int d, int f,
                             const moe_bf16* W1_local, const moe_bf16* W3_local, const moe_bf16* W2_local,
                             moe_bf16* h, const moe_bf16* x, int T, const moe_bf16* W1s, const moe_bf16* W3s,
                             const moe_bf16* W2s, int f_shared, moe_bf16* h_shared, moe_bf16* y_shared,
                             moe_bf16* const* y_perm_bufs, int64_t* row_dest, const void* ep_ws, size_t ep_ws_bytes,
                             moe_stream_t stream) {
    using namespace moe;
    int rc = ep_check(R, rank, E, d);
    if (rc != MOE_OK) return rc;
    MOE_REQUIRE(max_recv_rows >= 0 && f >= 64 && f % 64 == 0 && f_shared >= 0 && f_shared % 64 == 0, MOE_ERR_SHAPE);
    const bool shared = f_shared > 0;
    MOE_REQUIRE(ep_ws && y_perm_bufs && (max_recv_rows == 0 || (recv_x && W1_local && W3_local && W2_local && h &&
                                                                 row_dest)),
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!shared || (x && T >= 1 && W1s && W3s && W2s && h_shared && y_shared), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(recv_x) && aligned16(W1_local) && aligned16(W3_local) && aligned16(W2_local) &&
                    aligned16(h) && aligned16(x) && aligned16(W1s) && aligned16(W3s) && aligned16(W2s) &&
                    aligned16(h_shared) && aligned16(y_shared) && aligned16(ep_ws) && aligned16(row_dest),
                MOE_ERR_ALIGN);
    MOE_REQUIRE(ep_ws_bytes >= ep_bytes(R, E), MOE_ERR_WORKSPACE);
    EpDests dst;
    memset(&dst, 0, sizeof(dst));
    for (int q = 0; q < R; ++q) {
        MOE_REQUIRE(y_perm_bufs[q] && aligned16(y_perm_bufs[q]), MOE_ERR_INVALID_ARG);
        dst.base[q] = reinterpret_cast<char*>(y_perm_bufs[q]);
    }
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const EpView v = ep_view(const_cast<void*>(ep_ws), R, E);
    const int El = E / R;
    if (max_recv_rows > 0) {
        const int bx = std::max(1, std::min(8, (2 * di->sms + E - 1) / E));
        ep_row_dest_kernel<<<dim3(bx, E), 256, 0, s>>>(v.back, E, El, dst, (long long)d * 2,
                                                      reinterpret_cast<long long*>(row_dest));
        if ((rc = launch_status()) != MOE_OK) return rc;
    }
    FfnArgs a;
    memset(&a, 0, sizeof(a));
    a.x_perm = recv_x;
    a.max_rows = max_recv_rows;
    a.offsets = max_recv_rows ? v.exp_off : nullptr;
    a.mprefix = v.exp_tiles;
    a.E = El;
    a.d = d;
    a.f = f;
    a.W1 = W1_local; a.W3 = W3_local; a.W2 = W2_local;
    a.h = h;
    a.y_perm = reinterpret_cast<moe_bf16*>(dst.base[rank]);   // only for the tensor-map checks: rows go by row_dest
    a.y_row_addr = reinterpret_cast<const long long*>(row_dest);
    a.x = x; a.T = T; a.f_shared = f_shared; a.W1s = W1s; a.W3s = W3s; a.W2s = W2s;
    a.h_shared = h_shared; a.y_shared = y_shared;
    a.pair = use_pair_tiles(max_recv_rows, El);
    if (max_recv_rows == 0 && !shared) return MOE_OK;
    return run_expert_ffn(di, a, s);
}

int moe_update_bias(const int32_t* counts_raw, int E, int64_t capacity, float* bias, moe_stream_t stream) {
    MOE_REQUIRE(E >= 1 && E <= 1024, MOE_ERR_SHAPE);
    MOE_REQUIRE(capacity > 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(counts_raw && bias, MOE_ERR_INVALID_ARG);
    DeviceInfo* di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    update_bias_kernel<<<(E + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(counts_raw, E,
                                                                                      (long long)capacity, bias);
    return launch_status();
}

int moe_selftest_wait_timeout(moe_stream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    return launch_status();
}

int moe_get_error(moe_stream_t stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_moe_error, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_moe_error, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return v;
}

const char* moe_strerror(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_SHAPE: return "unsupported shape";
        case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_CHECK: return "device check failed (non-finite score or bad offsets)";
        case MOE_ERR_DEVICE: return "device is not sm_100";
        default: return "unknown status";
    }
}

}  // extern "C"

// The host-buffer pipeline and the no-allocation variant of moe_permute share this
// translation unit.
#include "pipeline.cuh"
#include "moe_noalloc.cu"
