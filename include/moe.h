/*
 * moe.h - C ABI of the B200 (sm_100a) MoE layer forward.
 *
 * The layer (Router -> Permutation -> Expert GEMM -> Combine) as the pages define it:
 *   [EP-KV]  "MoE 推理中的 Expert Parallel、KV Cache 与大规模专家并行架构解析"
 *            §1 (FFN with a SwiGLU gate), §2 (router + top-k experts + weighted combine,
 *            y = g5 E5(x) + g18 E18(x)), §7 (restore token order and aggregate),
 *            §8 (count, sort and pack tokens by expert, grouped GEMM), §10 (data path).
 *   [EP-DS3] "MoE 推理架构深度实战：从 Expert Parallelism 到 DeepSeek-V3 的工程落地"
 *            §2.1 router code (gate Linear without bias, softmax, top-k, renormalise,
 *            per-expert bias, bincount, capacity int(tokens/experts*factor)),
 *            §3.1 (sort the routing by expert id).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers to row-major, contiguous buffers that the
 *     caller owns (allocates and frees).  Pointers must be 16-byte aligned.
 *   - bf16 tensors are passed as moe_bf16 (the 16-bit pattern of a bfloat16).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *     and runs asynchronously.  The library never allocates device memory, never
 *     frees it and never synchronises, except moe_get_error().
 *   - The return value is a HOST-side status: argument validation and launch errors.
 *     Faults detected on the device (a non-finite router score, a bounded wait that
 *     ran out) are recorded in a per-device error word read by moe_get_error().
 *   - Shapes: 1 <= T, d % 64 == 0, f % 64 == 0, 1 <= k <= 32, k <= E <= 1024,
 *     T*k < 2^31.  A violation returns MOE_ERR_SHAPE and launches nothing.
 *   - Counts, offsets and the permutation stay on the device; no call reads them back,
 *     so a sequence of calls can be captured into a CUDA graph.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;   /* bit pattern of one bfloat16 */
typedef void* moe_stream_t;  /* cudaStream_t */

enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1, /* null pointer where one is required, bad enum value */
    MOE_ERR_SHAPE = -2,       /* shape outside the supported range */
    MOE_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
    MOE_ERR_WORKSPACE = -4,   /* ws_bytes smaller than moe_workspace_bytes() */
    MOE_ERR_CUDA = -5,        /* a CUDA runtime / driver call failed */
    MOE_ERR_TIMEOUT = -6,     /* device: a bounded wait inside a kernel ran out */
    MOE_ERR_CHECK = -7,       /* device: non-finite router score or inconsistent offsets */
    MOE_ERR_DEVICE = -8       /* the current device is not sm_100 */
};

enum moe_cap_mode {
    MOE_CAP_NONE = 0,           /* no capacity limit */
    MOE_CAP_PER_TOKEN = 1,      /* C = int(T / E * factor): the router's get_expert_capacity, [EP-DS3] §2.1 */
    MOE_CAP_PER_ASSIGNMENT = 2  /* C = int(T * k / E * factor): one slot per routed assignment */
};

/*
 * Capacity per expert, computed in double and truncated toward zero like Python's int()
 * ([EP-DS3] §2.1, capacity = int(num_tokens / num_experts * factor)).
 * Returns -1 (unlimited) for MOE_CAP_NONE or an unknown mode.
 */
int64_t moe_capacity(int T, int E, int k, double capacity_factor, int cap_mode);

/*
 * Bytes of device workspace that moe_layer_forward() needs for these shapes
 * (f_shared = 0: no shared expert).  The same size also covers moe_route(),
 * moe_permute() and moe_expert_ffn() for the same T, d, E, k, f.
 * Writes *bytes; returns MOE_OK or MOE_ERR_SHAPE / MOE_ERR_INVALID_ARG.
 */
int moe_workspace_bytes(int T, int d, int E, int k, int f, int f_shared, size_t* bytes);

/*
 * Router ([EP-DS3] §2.1 steps 1-4): logits = x Wg^T (fp32 accumulate on tensor cores),
 * then per token the k largest keys logit_e + bias_e (ties -> lower e, slots in
 * descending key order), and weights w_j = softmax(logits)_idx_j / sum over the k
 * selected, from the UNBIASED logits (the bias steers selection only).
 *   x         [T, d] bf16           hidden states (ignored if logits_in != NULL)
 *   Wg        [E, d] bf16           router weight (ignored if logits_in != NULL)
 *   bias      [E] fp32 or NULL      per-expert selection bias
 *   logits_in [T, E] fp32 or NULL   route these scores instead of computing x Wg^T
 *   logits_out[T, E] fp32 or NULL   receives the computed logits
 *   idx       [T, k] int32          selected experts
 *   w         [T, k] fp32           routing weights
 *   ws / ws_bytes                   workspace (moe_workspace_bytes)
 * Non-finite keys set MOE_ERR_CHECK in the device error word.
 */
int moe_route(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const float* logits_in,
              int T, int d, int E, int k, float* logits_out, int32_t* idx, float* w,
              void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Dispatch ([EP-KV] §8 count / sort / pack; [EP-DS3] §2.1 bincount + capacity, §3.1 sort by
 * expert id): per-expert histogram, capacity in token order (per expert the first
 * `capacity` assignments by ascending token index are kept; capacity < 0 = unlimited),
 * exclusive scan, and a stable permutation of the kept assignments into contiguous
 * per-expert row blocks.
 *   x          [T, d] bf16           hidden states
 *   idx        [T, k] int32          experts per token (distinct within a token, in [0, E))
 *   counts_raw [E] int32             assignments per expert before the capacity limit
 *   counts     [E] int32             kept assignments per expert
 *   offsets    [E+1] int32           exclusive scan of counts; offsets[E] = N kept rows
 *   dest       [T, k] int32          row of (t, j) in x_perm, or -1 if dropped
 *   src_token  [T*k] int32           src_token[r] = token of row r, for r < N
 *   x_perm     [T*k, d] bf16         x_perm[dest[t,j]] = x[t]; rows >= N untouched
 */
int moe_permute(const moe_bf16* x, const int32_t* idx, int T, int d, int E, int k, int64_t capacity,
                int32_t* counts_raw, int32_t* counts, int32_t* offsets, int32_t* dest, int32_t* src_token,
                moe_bf16* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute() for callers that cannot allocate device memory.  No counterpart on the
 * pages: it exists because some callers have no way to allocate at the point of the call
 * (a plugin inside a framework that owns all device memory, an engine whose memory plan
 * is fixed at start-up, a program that must not call cudaMalloc, which can synchronise
 * the device).  Same arguments and results as moe_permute() minus the workspace: the
 * scratch lives in a fixed array of MOE_NOALLOC_SCRATCH_BYTES compiled into the library,
 * which every GPU that loads the library holds until exit.
 *   - Sizes whose scratch, ceil(T/256)*E*4 + T*k*4 + (E+1)*4 bytes (each part rounded up
 *     to 256), exceeds MOE_NOALLOC_SCRATCH_BYTES return MOE_ERR_WORKSPACE; nothing runs.
 *   - The first call on a device, with that device current, looks up the array's device
 *     address (cudaGetSymbolAddress) and keeps it for the life of the process; make that
 *     first call before any stream capture.  A cudaDeviceReset() (or anything else that
 *     tears down the device's primary context) makes the kept address stale: do not call
 *     this entry point on that device again in the same process.
 *   - Calls on one device share the array: calls whose kernels overlap on the GPU race.
 *   - Allocates and frees nothing.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (4u << 20)
int moe_permute_noalloc(const moe_bf16* x, const int32_t* idx, int T, int d, int E, int k, int64_t capacity,
                        int32_t* counts_raw, int32_t* counts, int32_t* offsets, int32_t* dest,
                        int32_t* src_token, moe_bf16* x_perm, moe_stream_t stream);

/*
 * Experts ([EP-KV] §1 and §8): for every expert e, on rows [offsets[e], offsets[e+1]) of x_perm,
 *   h = bf16( silu(x_perm W1_e^T) * (x_perm W3_e^T) ),  y_perm = bf16( h W2_e^T ),
 * two grouped GEMMs on the tcgen05 tensor cores (fp32 accumulate in tensor memory),
 * SwiGLU fused into the first one's epilogue.  silu(a) = a / (1 + e^-a).
 *   x_perm   [max_rows, d] bf16      permuted hidden states (max_rows >= offsets[E], usually T*k)
 *   offsets  [E+1] int32 (device)    per-expert row ranges
 *   W1, W3   [E, f, d] bf16          gate / up projections
 *   W2       [E, d, f] bf16          down projection
 *   h        [max_rows, f] bf16      intermediate (written for rows < offsets[E])
 *   y_perm   [max_rows, d] bf16      expert outputs
 */
int moe_expert_ffn(const moe_bf16* x_perm, const int32_t* offsets, int max_rows, int E, int d, int f,
                   const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2,
                   moe_bf16* h, moe_bf16* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Combine ([EP-KV] §2 weighted sum, §7 restore order and aggregate):
 *   out[t] = bf16( sum_{j = 0..k-1, dest[t,j] >= 0} w[t,j] * y_perm[dest[t,j]]  (+ y_shared[t]) )
 * accumulated in fp32 in slot order j = 0..k-1, the shared expert added last with
 * weight 1; no atomics, so the result is deterministic.
 *   y_shared [T, d] bf16 or NULL
 */
int moe_combine(const moe_bf16* y_perm, const int32_t* dest, const float* w, const moe_bf16* y_shared,
                int T, int d, int k, moe_bf16* out, moe_stream_t stream);

/*
 * The whole layer: moe_route -> moe_permute -> moe_expert_ffn (+ the shared expert, run
 * in the same grouped-GEMM launches on all T tokens) -> moe_combine.
 *   W1s, W3s [f_shared, d], W2s [d, f_shared] bf16, all NULL and f_shared = 0 for none
 *   ([EP-KV] §3: routed and shared experts side by side).
 *   capacity = moe_capacity(T, E, k, capacity_factor, cap_mode).
 *   out [T, d] bf16.
 * Intermediates live in the workspace (layout: moe_workspace_layout()).
 */
int moe_layer_forward(const moe_bf16* x, const moe_bf16* Wg, const float* bias,
                      const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2,
                      const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s, int f_shared,
                      int T, int d, int E, int k, int f, double capacity_factor, int cap_mode,
                      moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Optional stage markers for measurement.  Each non-NULL member is a cudaEvent_t that
 * moe_layer_forward_ex() records on `stream` at the boundary it names; NULL members are
 * skipped.  Recording adds no work to the layer.
 */
typedef struct moe_stage_events {
    void* route;     /* before the router GEMM */
    void* topk;      /* before the top-k / softmax kernel */
    void* permute;   /* before the histogram / scan / scatter / gather kernels */
    void* gate_up;   /* before the first grouped GEMM (W1/W3 + SwiGLU) */
    void* down;      /* before the second grouped GEMM (W2) */
    void* combine;   /* before the combine kernel */
    void* end;       /* after the combine kernel */
    void* cache;     /* before the expert cache plan / copy kernels (moe_layer_forward_cached only) */
    void* gemm1;     /* fp8-activation layers: after quantising GEMM1's rows, before its kernel */
    void* gemm2;     /* fp8-activation layers: after quantising h, before GEMM2's kernel */
    void* copy_start;  /* cached layers: before the expert copy kernel, on the copy stream */
    void* copy_end;    /* cached layers: after the expert copy kernel, on the copy stream */
} moe_stage_events;

/* moe_layer_forward() with optional stage markers (events may be NULL). */
int moe_layer_forward_ex(const moe_bf16* x, const moe_bf16* Wg, const float* bias,
                         const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2,
                         const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s, int f_shared,
                         int T, int d, int E, int k, int f, double capacity_factor, int cap_mode,
                         moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                         const moe_stage_events* events);

/*
 * The layer with fp8 expert weights (the pages' low-bit quantization option for the expert
 * weights, "low-bit expert weights for decode streaming"): every weight is one fp8 e4m3 byte
 * q ("fn" encoding: no infinities, max 448) and every output row one fp32 scale, so the
 * expert weight W[n, i] = e4m3(q[n, i]) * s[n].  The decode layer streams half the bytes of
 * bf16 weights.  Everything else (router in bf16, routing, permutation, combine, rounding of
 * h / y / out to bf16) is as in moe_layer_forward().
 *   W1q, W3q [E, f, d] uint8, s1, s3 [E, f] fp32      gate / up
 *   W2q [E, d, f] uint8, s2 [E, d] fp32                 down
 *   W1sq, W3sq [f_shared, d], s1s, s3s [f_shared], W2sq [d, f_shared], s2s [d]: shared expert
 *   (all NULL with f_shared = 0).  Same workspace as moe_layer_forward().
 */
int moe_layer_forward_w8(const moe_bf16* x, const moe_bf16* Wg, const float* bias,
                         const uint8_t* W1q, const float* s1, const uint8_t* W3q, const float* s3,
                         const uint8_t* W2q, const float* s2,
                         const uint8_t* W1sq, const float* s1s, const uint8_t* W3sq, const float* s3s,
                         const uint8_t* W2sq, const float* s2s, int f_shared,
                         int T, int d, int E, int k, int f, double capacity_factor, int cap_mode,
                         moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                         const moe_stage_events* events);

/*
 * One global token batch sharded over G ranks (one process per GPU), with a capacity limit.
 * Token-order dropping is global: rank r's tokens come after those of ranks 0..r-1, so an
 * expert may keep only capacity - (its assignments on earlier ranks) of rank r's.  The one
 * exchange this needs happens between two calls:
 *   1. moe_layer_route_count(): router + top-k + per-expert histogram of this rank's batch;
 *      counts_raw (workspace offset off[3] of moe_workspace_layout, [E] int32) is then valid.
 *   2. the caller all-gathers every rank's counts_raw into all_counts [G, E] (rank-major),
 *      e.g. with ncclAllGather, and moe_fill_base() turns it into this rank's
 *      fill_base[e] = sum_{g < rank} all_counts[g, e].
 *   3. moe_layer_finish(): permutation with the global capacity (e.g. moe_capacity(G*T, ...))
 *      and fill_base, then experts (+ shared) and combine, on the same workspace.
 * With fill_base = NULL, moe_layer_finish() after moe_layer_route_count() equals
 * moe_layer_forward() with that capacity.  Same shapes, pointers and workspace rules as
 * moe_layer_forward(); x must be the same tensor in both calls.
 */
int moe_layer_route_count(const moe_bf16* x, const moe_bf16* Wg, const float* bias, int f_shared,
                          int T, int d, int E, int k, int f, void* ws, size_t ws_bytes, moe_stream_t stream);
int moe_fill_base(const int32_t* all_counts, int G, int rank, int E, int32_t* fill_base, moe_stream_t stream);
int moe_layer_finish(const moe_bf16* x, const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2,
                     const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s, int f_shared,
                     int T, int d, int E, int k, int f, int64_t capacity, const int32_t* fill_base,
                     moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Selection bias from the overflow of the last batch ([EP-DS3] §2.1, the router's expert_bias
 * update, applied between batches at inference):
 *   bias[e] = -clamp((counts_raw[e] - capacity) / capacity, -1, 1)      (fp32, IEEE division)
 * An expert routed more than `capacity` times gets a negative bias (fewer later tokens pick
 * it), an idle one up to +1.  The page's comment states that sign; the formula it prints
 * omits the minus.  Pass the result as `bias` of the next moe_route / moe_layer_forward.
 *   counts_raw [E] int32 (device), e.g. the counts_raw that moe_permute wrote
 *   capacity   > 0, e.g. moe_capacity(T, E, k, factor, MOE_CAP_PER_TOKEN)
 *   bias       [E] fp32 (device), overwritten
 */
int moe_update_bias(const int32_t* counts_raw, int E, int64_t capacity, float* bias, moe_stream_t stream);

/*
 * Host-buffer pipeline: hidden-state batches in (pinned) host memory run through the layer
 * with the copy of the next batch to the device and of the previous result back to the
 * host overlapping the current batch's layer (two device slots, three streams: copy in,
 * layer, copy out).  Layer parameters are fixed per pipeline; all pointers in the params
 * are device pointers as for moe_layer_forward(), except nothing here is a batch.
 *   moe_pipeline_bytes():   device memory the pipeline needs (2 input + 2 output slots of
 *                           T*d bf16 and one layer workspace); the caller allocates it.
 *   moe_pipeline_create():  binds the params and that memory; creates streams and events.
 *   moe_pipeline_submit():  enqueues one batch: x_host [T,d] -> layer -> out_host [T,d].
 *                           Returns at once; both host buffers must stay valid (and x_host
 *                           unchanged) until moe_pipeline_sync().  Pinned memory makes the
 *                           copies asynchronous.
 *   moe_pipeline_sync():    waits for every submitted batch.
 *   moe_pipeline_streams(): the three streams (e.g. to record timing events).
 *   moe_pipeline_destroy(): syncs, then releases streams and events (not the caller's memory).
 */
typedef struct moe_pipeline_params {
    const moe_bf16 *Wg, *W1, *W3, *W2;          /* routed experts and router */
    const moe_bf16 *W1s, *W3s, *W2s;            /* shared expert, NULL if f_shared == 0 */
    const float* bias;                          /* selection bias [E] or NULL */
    int T, d, E, k, f, f_shared;
    double capacity_factor;
    int cap_mode;
} moe_pipeline_params;
typedef struct moe_pipeline moe_pipeline;
int moe_pipeline_bytes(int T, int d, int E, int k, int f, int f_shared, size_t* bytes);
int moe_pipeline_create(const moe_pipeline_params* params, void* dev_mem, size_t dev_bytes, moe_pipeline** out);
int moe_pipeline_submit(moe_pipeline* pipeline, const moe_bf16* x_host, moe_bf16* out_host);
int moe_pipeline_sync(moe_pipeline* pipeline);
int moe_pipeline_streams(moe_pipeline* pipeline, moe_stream_t* h2d, moe_stream_t* compute, moe_stream_t* d2h);
int moe_pipeline_destroy(moe_pipeline* pipeline);

/*
 * The permutation alone, in the layer workspace (counts, offsets, dest, src_token, x_perm at
 * their moe_workspace_layout() offsets): histogram, capacity with fill_base (as in
 * moe_layer_finish), stable scatter and the gather of x_perm.  Needs the routing of
 * moe_layer_route_count() in the same workspace.  Used by the expert-parallel path.
 */
int moe_layer_permute(const moe_bf16* x, int f_shared, int T, int d, int E, int k, int f, int64_t capacity,
                      const int32_t* fill_base, void* ws, size_t ws_bytes, moe_stream_t stream);
/* moe_layer_permute() without the row gather: counts, offsets, dest and src_token only; x_perm is
 * left unwritten (for moe_ep_dispatch_gather(), which moves x's rows itself). */
int moe_layer_permute_indices(const moe_bf16* x, int f_shared, int T, int d, int E, int k, int f, int64_t capacity,
                              const int32_t* fill_base, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Expert parallelism: the E routed experts are split over R ranks, rank r holding experts
 * [r El, (r + 1) El), El = E / R (uniform contiguous assignment).  [EP-KV] "MoE 推理中的 Expert
 * Parallel、KV Cache 与大规模专家并行架构解析" sections 6-7: a layer sends each token's hidden
 * state to the ranks of its experts and the expert outputs back to the token's rank, which
 * combines them; all-to-all-v, point-to-point copies or fused kernels are all valid ways to move
 * them.  [EP-DS3] section 3.1 (_assign_experts) gives the contiguous split.
 *
 * Per rank, per layer call (all asynchronous on `stream`):
 *   1. moe_layer_route_count()                 routing and raw counts of the rank's T tokens
 *   2. all-gather of counts_raw -> all_counts_raw [R, E] int32 on every rank (the caller's
 *      collective; rank order = token order of the whole batch)
 *   3. moe_fill_base() + moe_layer_permute()  global-capacity keep decisions, x_perm
 *   4. moe_ep_plan()                           from all_counts_raw alone: the row ranges this
 *      rank sends and returns, and the groups of its local GEMM (into ep_ws)
 *      moe_ep_dispatch()                       puts this rank's x_perm rows of each expert into
 *      the receive buffer of the expert's rank, in expert-major order there (the rows of one
 *      local expert from all ranks are contiguous, in rank order), so each local expert is one
 *      GEMM group and its weights are read once
 *      (a caller with a collective library can move the rows with an all-to-all-v instead:
 *      rank r sends its rows of q's experts to q; they arrive source-major, and
 *      moe_ep_expert_ffn(source_major = 1) runs one segment per (source rank, local expert))
 *   5. a barrier (every rank's puts done before any rank reads its receive buffer)
 *   6. moe_ep_expert_ffn()                     local experts over the received rows + the
 *      shared expert on the rank's own tokens
 *   7. moe_ep_return()                         puts each result row back into the y_perm (layer
 *      workspace) of the rank it came from, at the row it had in that rank's x_perm
 *   8. a barrier, then moe_combine() with the rank's dest, w (layer workspace) and y_shared
 * The output equals the single-GPU layer over the whole batch (capacity counted over all ranks).
 *
 * Buffers: recv_bufs / y_perm_bufs are host arrays of R device addresses, one per rank, that
 * this device can write (peer-mapped buffers of other GPUs, or the same GPU's buffers when
 * ranks share a device).  A receive buffer holds max_recv_rows rows of d bf16 (>= the rows the
 * rank can receive: R * T * k bounds it).  ep_ws: moe_ep_workspace_bytes(E) bytes, 16-byte
 * aligned (moe_ep_workspace_bytes(R, E)), written by moe_ep_plan() and read by the later calls
 * on the same rank.
 * Errors: MOE_ERR_SHAPE unless 1 <= R <= 64, E % R == 0, E <= 1024, 0 <= rank < R.
 * moe_ep_expert_ffn: source_major = 0 after moe_ep_dispatch(), 1 after an all-to-all-v.
 */
int moe_ep_workspace_bytes(int R, int E, size_t* bytes);
/*
 * Byte offset inside ep_ws of the split table moe_ep_plan() writes: int32 [2, R], row 0 = rows
 * this rank sends to each rank q (its kept rows of q's experts), row 1 = rows it receives from
 * each rank s (s's kept rows of this rank's experts).  These are the split sizes of the two
 * all-to-all-v exchanges (dispatch: send / receive; return: the same rows swapped), computed on
 * the device with the rest of the plan.  MOE_ERR_SHAPE as for moe_ep_workspace_bytes().
 */
int moe_ep_splits_offset(int R, int E, size_t* offset);
int moe_ep_plan(const int32_t* all_counts_raw, int R, int rank, int E, int64_t capacity, int max_recv_rows,
                void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream);
int moe_ep_dispatch(const moe_bf16* x_perm, int R, int rank, int E, int d, moe_bf16* const* recv_bufs,
                    const void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream);
/*
 * moe_ep_dispatch() fused with the permutation's gather: after moe_layer_permute_indices() and
 * moe_ep_plan(), each kept row is copied from x (token src_token[r] for x_perm row r; src_token
 * is the layer workspace's) straight into the receive buffer of its expert's rank, at the row
 * moe_ep_dispatch() would have put it, so x_perm is never written or read.  Same receive layout
 * and errors as moe_ep_dispatch().
 */
int moe_ep_dispatch_gather(const moe_bf16* x, const int32_t* src_token, int R, int rank, int E, int d,
                           moe_bf16* const* recv_bufs, const void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream);
int moe_ep_expert_ffn(const moe_bf16* recv_x, int max_recv_rows, int source_major, int R, int rank, int E, int d,
                      int f,
                      const moe_bf16* W1_local, const moe_bf16* W3_local, const moe_bf16* W2_local, moe_bf16* h,
                      moe_bf16* y_recv, const moe_bf16* x, int T, const moe_bf16* W1s, const moe_bf16* W3s,
                      const moe_bf16* W2s, int f_shared, moe_bf16* h_shared, moe_bf16* y_shared, const void* ep_ws,
                      size_t ep_ws_bytes, moe_stream_t stream);
int moe_ep_return(const moe_bf16* y_recv, int R, int rank, int E, int d, moe_bf16* const* y_perm_bufs,
                  const void* ep_ws, size_t ep_ws_bytes, moe_stream_t stream);
/*
 * Steps 6 and 7 in one: moe_ep_expert_ffn() (expert-major receive buffer, after
 * moe_ep_dispatch()) whose second grouped GEMM stores every result row straight into the y_perm of
 * the rank the row came from, at the row it had there ([EP-KV] section 7: the combine-side
 * exchange fused into the expert computation), so the rows cross to the other GPUs while later
 * tiles are still being computed and no y_recv buffer or return copy is needed.  A small kernel
 * first writes the byte address of every received row's destination into row_dest
 * [max_recv_rows] int64 (device, 16-byte aligned, caller-owned scratch).  y_perm_bufs: as for
 * moe_ep_return().  The shared expert's output goes to y_shared as in moe_ep_expert_ffn().  The
 * results are the same bits as moe_ep_expert_ffn() + moe_ep_return().
 */
int moe_ep_expert_ffn_return(const moe_bf16* recv_x, int max_recv_rows, int R, int rank, int E, int d, int f,
                             const moe_bf16* W1_local, const moe_bf16* W3_local, const moe_bf16* W2_local,
                             moe_bf16* h, const moe_bf16* x, int T, const moe_bf16* W1s, const moe_bf16* W3s,
                             const moe_bf16* W2s, int f_shared, moe_bf16* h_shared, moe_bf16* y_shared,
                             moe_bf16* const* y_perm_bufs, int64_t* row_dest, const void* ep_ws, size_t ep_ws_bytes,
                             moe_stream_t stream);

/*
 * Peer buffers for the put exchange with one process per GPU ([EP-KV] section 7: point-to-point
 * copies into the other ranks' memory).  Each rank exports its receive buffer and its y_perm,
 * the ranks exchange the handles (any host channel: the caller's collective library), and each
 * rank imports the others' handles to get device addresses its put kernels can store to
 * (plain peer stores over NVLink; nothing else reads another GPU's memory).
 *   moe_ipc_export(ptr, handle)   handle: MOE_IPC_HANDLE_BYTES bytes (host) describing the device
 *                                 allocation that holds ptr and ptr's offset in it
 *   moe_ipc_import(handle, &ptr)  maps another process's exported allocation into this process
 *                                 (cudaIpcOpenMemHandle, peer access enabled lazily) and returns
 *                                 the address of the exported pointer; a process uses its own
 *                                 pointers for its own buffers (CUDA IPC maps other processes')
 *   moe_ipc_close(ptr, handle)    unmaps what moe_ipc_import returned for that handle
 * The exporter must keep the allocation alive until every importer has closed it.  Errors:
 * MOE_ERR_INVALID_ARG (null arguments, a pointer that is not device memory, a foreign blob),
 * MOE_ERR_CUDA (the runtime refused the export, import or close).  Synchronous host calls.
 */
#define MOE_IPC_HANDLE_BYTES 96
int moe_ipc_export(const void* ptr, void* handle);
int moe_ipc_import(const void* handle, void** ptr);
int moe_ipc_close(void* ptr, const void* handle);

/*
 * The layer with fp8 e4m3 weights AND fp8 activations: the weights as in moe_layer_forward_w8();
 * every activation row entering an expert GEMM (the token's hidden state, then h) is quantised
 * on its own, s_row = amax(|row|) / 448 in fp32 (1 for an all-zero row), codes
 * e4m3(fp32(x) / s_row) rounded to nearest even, saturating at 448 (the deployment page's
 * "w4afp8" option: low-bit weights with fp8 activations).  The expert GEMMs run fp8 x fp8 on
 * the tensor cores (tcgen05 kind::f8f6f4) with fp32 accumulation and scale each sum by
 * s_row * s_col before SwiGLU / the bf16 store.  Router, routing, permutation and combine as in
 * moe_layer_forward().  Workspace: moe_workspace_bytes_a8() (the layer workspace followed by the
 * quantised rows and their scales).  Shapes: d, f, f_shared multiples of 128 (MOE_ERR_SHAPE).
 * Each token row of x is quantised once and its codes written to its permuted rows (dest), so
 * the workspace's x_perm is not written by this layer.
 */
int moe_workspace_bytes_a8(int T, int d, int E, int k, int f, int f_shared, size_t* bytes);
int moe_layer_forward_w8a8(const moe_bf16* x, const moe_bf16* Wg, const float* bias,
                           const uint8_t* W1q, const float* s1, const uint8_t* W3q, const float* s3,
                           const uint8_t* W2q, const float* s2,
                           const uint8_t* W1sq, const float* s1s, const uint8_t* W3sq, const float* s3s,
                           const uint8_t* W2sq, const float* s2s, int f_shared,
                           int T, int d, int E, int k, int f, double capacity_factor, int cap_mode,
                           moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                           const moe_stage_events* events);

/*
 * Expert cache: the routed experts' weights live in page-locked host memory and HBM holds S
 * expert slots managed as an LRU.  [EP-DS3] "MoE 推理架构深度实战：从 Expert Parallelism 到
 * DeepSeek-V3 的工程落地", section 3.2 (expert cache and preloading): inactive experts are
 * kept in host memory, the experts a batch needs are loaded, the least recently used resident
 * expert is evicted when the slots are full.  Readings where the page's sketch is open:
 * recency is counted in batches (every expert a batch keeps at least one row for is stamped
 * with the batch number, hit or miss); misses are filled in ascending expert order, each into
 * the slot with the oldest stamp among the slots the batch does not use (empty slots first,
 * then ties to the lower slot).  The decision and the copies run on the device after the
 * batch's counts exist: no host round trip, capturable in a CUDA graph.
 *
 * State (caller-owned device memory, 16-byte aligned, moe_cache_state_bytes() bytes):
 *   off[0] moe_cache_counters   off[1] slot_of [E] int32 (-1 = host only)
 *   off[2] expert_in [S] int32 (-1 = empty)   off[3] stamp [S] int32 (batch of last use, -1)
 *   off[4] load_expert [S] int32   off[5] load_slot [S] int32 (the last batch's loads, in order)
 * moe_cache_reset() empties the cache (asynchronous on `stream`).
 */
typedef struct moe_cache_counters {
    int64_t step;        /* batches run through the cache */
    int64_t hits;        /* (batch, expert) pairs that found the expert resident */
    int64_t misses;      /* (batch, expert) pairs that loaded it */
    int64_t loads_last;  /* experts loaded by the last batch */
    int64_t reserved[4];
} moe_cache_counters;

/* Bytes of the cache state; MOE_ERR_SHAPE unless 1 <= S <= E <= 1024. */
int moe_cache_state_bytes(int E, int S, size_t* bytes);
int moe_cache_layout(int E, int S, size_t off[6]);
int moe_cache_reset(void* cache_state, int E, int S, moe_stream_t stream);

/*
 * moe_layer_forward() with the routed experts served from the cache.
 *   W1_src, W3_src [E, f, d], W2_src [E, d, f]: the weights; page-locked host memory
 *       (cudaHostAlloc / cudaHostRegister) read directly by the copy kernel, or device memory.
 *       Pageable host memory is rejected (MOE_ERR_INVALID_ARG).
 *   W1_slots, W3_slots [S, f, d], W2_slots [S, d, f]: device memory of the slots.
 *   S: slots; must be >= min(E, T*k) so that one batch always fits (else MOE_ERR_SHAPE).
 * Per batch, after the counts: the plan kernel updates the state and lists the loads, the copy
 * kernel brings those experts into their slots, the grouped GEMMs read expert e from slot
 * slot_of[e].  The copy overlaps compute ([EP-DS3] section 3.2): it runs on a copy stream of the
 * library's own (one per device, created on first use), forked from `stream` after the plan;
 * meanwhile both grouped GEMMs run on `stream` over the experts that were already resident (and
 * the shared expert), then `stream` waits for the copy and the GEMMs run over the loaded ones.
 * Cached-layer calls on one device share that copy stream, so their copies run one after
 * another.  The output is the same as moe_layer_forward() with W1/W3/W2 = the sources.
 * Device-side failure (a batch that needs more than S experts) sets MOE_ERR_CHECK.
 */
int moe_layer_forward_cached(const moe_bf16* x, const moe_bf16* Wg, const float* bias,
                             const moe_bf16* W1_src, const moe_bf16* W3_src, const moe_bf16* W2_src,
                             moe_bf16* W1_slots, moe_bf16* W3_slots, moe_bf16* W2_slots, int S,
                             void* cache_state, const moe_bf16* W1s, const moe_bf16* W3s, const moe_bf16* W2s,
                             int f_shared, int T, int d, int E, int k, int f, double capacity_factor,
                             int cap_mode, moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                             const moe_stage_events* events);

/*
 * The cached layer with fp8 expert weights (moe_layer_forward_w8's format): the sources hold
 * every expert's codes and row scales, the slots S experts' worth of each.  A miss copies half
 * the bytes of a bf16 expert over the host link.
 *   src:    W1q, W3q [E, f, d] uint8, W2q [E, d, f] uint8, s1, s3 [E, f], s2 [E, d] fp32;
 *           page-locked host memory or device memory
 *   slots:  the same arrays with S in place of E, device memory
 *   shared: the shared expert (W1q, W3q [f_shared, d], W2q [d, f_shared], s1, s3 [f_shared],
 *           s2 [d]), device memory, or NULL with f_shared = 0
 * Same state, workspace and checks as moe_layer_forward_cached().
 */
typedef struct moe_w8_experts {
    const uint8_t *W1q, *W3q, *W2q;
    const float *s1, *s3, *s2;
} moe_w8_experts;
typedef struct moe_w8_slots {
    uint8_t *W1q, *W3q, *W2q;
    float *s1, *s3, *s2;
} moe_w8_slots;
int moe_layer_forward_cached_w8(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_w8_experts* src,
                                const moe_w8_slots* slots, int S, void* cache_state, const moe_w8_experts* shared,
                                int f_shared, int T, int d, int E, int k, int f, double capacity_factor, int cap_mode,
                                moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream,
                                const moe_stage_events* events);

/*
 * The host-buffer pipeline (moe_pipeline_*) over the fp8 layers: the same two device slots,
 * three streams and overlapped copies, with moe_layer_forward_w8() (activations_fp8 = 0) or
 * moe_layer_forward_w8a8() (activations_fp8 = 1) as the layer.  params gives the router (Wg,
 * bias), the shapes and the capacity; its W1..W2s are ignored.  routed / shared: the fp8 codes
 * and row scales (shared may be NULL when f_shared == 0).  moe_pipeline_bytes_w8(): device
 * memory to pass (2 input + 2 output slots and that layer's workspace).  submit, sync, streams
 * and destroy are the moe_pipeline_* calls above.  Errors as moe_pipeline_create(), plus
 * MOE_ERR_INVALID_ARG for missing fp8 arrays; shapes are checked by the layer at submit.
 */
int moe_pipeline_bytes_w8(int T, int d, int E, int k, int f, int f_shared, int activations_fp8, size_t* bytes);
int moe_pipeline_create_w8(const moe_pipeline_params* params, const moe_w8_experts* routed,
                           const moe_w8_experts* shared, int activations_fp8, void* dev_mem, size_t dev_bytes,
                           moe_pipeline** out);

/*
 * Byte offsets of the intermediates that moe_layer_forward() leaves in its workspace,
 * so that a caller (a test) can read them after the call:
 *   off[0] logits [T,E] fp32   off[1] idx [T,k] int32   off[2] w [T,k] fp32
 *   off[3] counts_raw [E]      off[4] counts [E]        off[5] offsets [E+1]
 *   off[6] dest [T,k]          off[7] src_token [T*k]   off[8] x_perm [T*k,d] bf16
 *   off[9] h [T*k,f] bf16      off[10] y_perm [T*k,d]   off[11] y_shared [T,d] bf16
 *   off[12] h_shared [T,f_shared] bf16
 * Returns MOE_OK or a shape error.
 */
int moe_workspace_layout(int T, int d, int E, int k, int f, int f_shared, size_t off[13]);

/*
 * Synchronises `stream`, returns the first device-side error recorded on the current
 * device since the last call (MOE_OK if none) and clears it.  The error word is shared
 * by all streams of the device.
 */
int moe_get_error(moe_stream_t stream);

/*
 * Failure-detection self-test: enqueues one kernel whose single bounded wait on an mbarrier
 * can never be satisfied.  After the wait limit (2 s) the kernel records MOE_ERR_TIMEOUT in the
 * device error word and returns; the next moe_get_error() reports it and the device stays
 * usable.  Returns the host launch status.
 */
int moe_selftest_wait_timeout(moe_stream_t stream);

/* Static text for a status code. */
const char* moe_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
