// pipeline.cuh - host-buffer pipeline: batches of hidden states in pinned host memory run
// through the layer with their copies overlapped.
//
// Two device slots (input + output rows) and three streams: the copy of batch i+1 to the
// device and the copy of batch i-1 back to the host run while batch i runs the layer.
//   h2d stream:     wait (slot's previous layer done) -> copy x_host -> x_dev[slot]
//   compute stream: wait (x copied, slot's previous output read back) -> layer -> out_dev[slot]
//   d2h stream:     wait (layer done) -> copy out_dev[slot] -> out_host
// All layers run on the one compute stream, so they share one workspace.  The device memory
// (2 x (x + out) + workspace) is the caller's; the pipeline owns only streams and events.

#pragma once

#include <cstring>
#include <new>

namespace moe {

// weights: 0 = bf16 (moe_layer_forward), 1 = fp8 weights (moe_layer_forward_w8),
// 2 = fp8 weights and activations (moe_layer_forward_w8a8)
enum { PIPE_BF16 = 0, PIPE_W8 = 1, PIPE_W8A8 = 2 };

struct Pipeline {
    moe_pipeline_params prm;
    int weights;
    moe_w8_experts q, qs;       // fp8 routed and shared experts (weights != PIPE_BF16)
    char* x_dev[2];
    char* out_dev[2];
    void* ws;
    size_t ws_bytes;
    cudaStream_t h2d, compute, d2h;
    cudaEvent_t h2d_done[2], layer_done[2], d2h_done[2];
    long long submitted;
};

inline size_t pipeline_io_bytes(int T, int d) { return align256((size_t)T * d * 2); }

}  // namespace moe

extern "C" {

int moe_pipeline_bytes(int T, int d, int E, int k, int f, int f_shared, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    size_t ws = 0;
    int rc = moe_workspace_bytes(T, d, E, k, f, f_shared, &ws);
    if (rc != MOE_OK) return rc;
    *bytes = 4 * moe::pipeline_io_bytes(T, d) + moe::align256(ws);
    return MOE_OK;
}

int moe_pipeline_bytes_w8(int T, int d, int E, int k, int f, int f_shared, int activations_fp8, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    size_t ws = 0;
    int rc = activations_fp8 ? moe_workspace_bytes_a8(T, d, E, k, f, f_shared, &ws)
                             : moe_workspace_bytes(T, d, E, k, f, f_shared, &ws);
    if (rc != MOE_OK) return rc;
    *bytes = 4 * moe::pipeline_io_bytes(T, d) + moe::align256(ws);
    return MOE_OK;
}

namespace {

int pipeline_create(const moe_pipeline_params* prm, int weights, const moe_w8_experts* q, const moe_w8_experts* qs,
                    void* dev_mem, size_t dev_bytes, moe_pipeline** out) {
    using namespace moe;
    if (!prm || !dev_mem || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(dev_mem)) return MOE_ERR_ALIGN;
    size_t need = 0;
    int rc = weights == PIPE_BF16
                 ? moe_pipeline_bytes(prm->T, prm->d, prm->E, prm->k, prm->f, prm->f_shared, &need)
                 : moe_pipeline_bytes_w8(prm->T, prm->d, prm->E, prm->k, prm->f, prm->f_shared,
                                         weights == PIPE_W8A8, &need);
    if (rc != MOE_OK) return rc;
    if (dev_bytes < need) return MOE_ERR_WORKSPACE;
    if (!prm->Wg) return MOE_ERR_INVALID_ARG;
    if (weights == PIPE_BF16 && !(prm->W1 && prm->W3 && prm->W2)) return MOE_ERR_INVALID_ARG;
    if (weights != PIPE_BF16 && !(q && q->W1q && q->W3q && q->W2q && q->s1 && q->s3 && q->s2)) return MOE_ERR_INVALID_ARG;
    if (weights != PIPE_BF16 && prm->f_shared > 0 &&
        !(qs && qs->W1q && qs->W3q && qs->W2q && qs->s1 && qs->s3 && qs->s2))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    Pipeline* pl = new (std::nothrow) Pipeline;
    if (!pl) return MOE_ERR_INVALID_ARG;
    memset(pl, 0, sizeof(Pipeline));
    pl->prm = *prm;
    pl->weights = weights;
    if (weights != PIPE_BF16) {
        pl->q = *q;
        if (prm->f_shared > 0) pl->qs = *qs;
    }
    char* base = static_cast<char*>(dev_mem);
    const size_t io = pipeline_io_bytes(prm->T, prm->d);
    pl->x_dev[0] = base;
    pl->x_dev[1] = base + io;
    pl->out_dev[0] = base + 2 * io;
    pl->out_dev[1] = base + 3 * io;
    pl->ws = base + 4 * io;
    pl->ws_bytes = dev_bytes - 4 * io;
    bool ok = cudaStreamCreateWithFlags(&pl->h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&pl->compute, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&pl->d2h, cudaStreamNonBlocking) == cudaSuccess;
    for (int s = 0; s < 2 && ok; ++s)
        ok = cudaEventCreateWithFlags(&pl->h2d_done[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&pl->layer_done[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&pl->d2h_done[s], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        moe_pipeline_destroy(reinterpret_cast<moe_pipeline*>(pl));
        return MOE_ERR_CUDA;
    }
    *out = reinterpret_cast<moe_pipeline*>(pl);
    return MOE_OK;
}

}  // namespace

int moe_pipeline_create(const moe_pipeline_params* prm, void* dev_mem, size_t dev_bytes, moe_pipeline** out) {
    return pipeline_create(prm, moe::PIPE_BF16, nullptr, nullptr, dev_mem, dev_bytes, out);
}

int moe_pipeline_create_w8(const moe_pipeline_params* prm, const moe_w8_experts* routed, const moe_w8_experts* shared,
                           int activations_fp8, void* dev_mem, size_t dev_bytes, moe_pipeline** out) {
    return pipeline_create(prm, activations_fp8 ? moe::PIPE_W8A8 : moe::PIPE_W8, routed, shared, dev_mem, dev_bytes,
                           out);
}

int moe_pipeline_submit(moe_pipeline* handle, const moe_bf16* x_host, moe_bf16* out_host) {
    using namespace moe;
    Pipeline* pl = reinterpret_cast<Pipeline*>(handle);
    if (!pl || !x_host || !out_host) return MOE_ERR_INVALID_ARG;
    const moe_pipeline_params& p = pl->prm;
    const int s = (int)(pl->submitted & 1);
    const size_t bytes = (size_t)p.T * p.d * 2;
    // h2d: the slot's input is free once the layer that read it (two batches ago) is done
    if (pl->submitted >= 2 && cudaStreamWaitEvent(pl->h2d, pl->layer_done[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(pl->x_dev[s], x_host, bytes, cudaMemcpyHostToDevice, pl->h2d) != cudaSuccess ||
        cudaEventRecord(pl->h2d_done[s], pl->h2d) != cudaSuccess)
        return MOE_ERR_CUDA;
    // compute: after the copy in, and after the slot's previous output went back to the host
    if (cudaStreamWaitEvent(pl->compute, pl->h2d_done[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (pl->submitted >= 2 && cudaStreamWaitEvent(pl->compute, pl->d2h_done[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
    const moe_bf16* xd = reinterpret_cast<const moe_bf16*>(pl->x_dev[s]);
    moe_bf16* od = reinterpret_cast<moe_bf16*>(pl->out_dev[s]);
    int rc;
    if (pl->weights == PIPE_BF16) {
        rc = moe_layer_forward(xd, p.Wg, p.bias, p.W1, p.W3, p.W2, p.W1s, p.W3s, p.W2s, p.f_shared, p.T, p.d, p.E, p.k,
                               p.f, p.capacity_factor, p.cap_mode, od, pl->ws, pl->ws_bytes, pl->compute);
    } else {
        const moe_w8_experts& q = pl->q;
        const moe_w8_experts& qs = pl->qs;
        auto call = pl->weights == PIPE_W8A8 ? moe_layer_forward_w8a8 : moe_layer_forward_w8;
        rc = call(xd, p.Wg, p.bias, q.W1q, q.s1, q.W3q, q.s3, q.W2q, q.s2, qs.W1q, qs.s1, qs.W3q, qs.s3, qs.W2q,
                  qs.s2, p.f_shared, p.T, p.d, p.E, p.k, p.f, p.capacity_factor, p.cap_mode, od, pl->ws,
                  pl->ws_bytes, pl->compute, nullptr);
    }
    if (rc != MOE_OK) return rc;
    if (cudaEventRecord(pl->layer_done[s], pl->compute) != cudaSuccess) return MOE_ERR_CUDA;
    // d2h: after the layer
    if (cudaStreamWaitEvent(pl->d2h, pl->layer_done[s], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_host, pl->out_dev[s], bytes, cudaMemcpyDeviceToHost, pl->d2h) != cudaSuccess ||
        cudaEventRecord(pl->d2h_done[s], pl->d2h) != cudaSuccess)
        return MOE_ERR_CUDA;
    ++pl->submitted;
    return MOE_OK;
}

int moe_pipeline_sync(moe_pipeline* handle) {
    moe::Pipeline* pl = reinterpret_cast<moe::Pipeline*>(handle);
    if (!pl) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(pl->h2d) != cudaSuccess || cudaStreamSynchronize(pl->compute) != cudaSuccess ||
        cudaStreamSynchronize(pl->d2h) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_pipeline_streams(moe_pipeline* handle, moe_stream_t* h2d, moe_stream_t* compute, moe_stream_t* d2h) {
    moe::Pipeline* pl = reinterpret_cast<moe::Pipeline*>(handle);
    if (!pl) return MOE_ERR_INVALID_ARG;
    if (h2d) *h2d = pl->h2d;
    if (compute) *compute = pl->compute;
    if (d2h) *d2h = pl->d2h;
    return MOE_OK;
}

int moe_pipeline_destroy(moe_pipeline* handle) {
    moe::Pipeline* pl = reinterpret_cast<moe::Pipeline*>(handle);
    if (!pl) return MOE_OK;
    moe_pipeline_sync(handle);
    for (int s = 0; s < 2; ++s) {
        if (pl->h2d_done[s]) cudaEventDestroy(pl->h2d_done[s]);
        if (pl->layer_done[s]) cudaEventDestroy(pl->layer_done[s]);
        if (pl->d2h_done[s]) cudaEventDestroy(pl->d2h_done[s]);
    }
    if (pl->h2d) cudaStreamDestroy(pl->h2d);
    if (pl->compute) cudaStreamDestroy(pl->compute);
    if (pl->d2h) cudaStreamDestroy(pl->d2h);
    delete pl;
    return MOE_OK;
}

}  // extern "C"
