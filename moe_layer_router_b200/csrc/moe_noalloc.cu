// moe_noalloc.cu - moe_permute_noalloc(): the permutation stage for callers that cannot
// allocate device memory.
//
// Why it exists.  moe_permute() needs a small scratch area (per-block expert counts, the
// stable rank of every assignment, the GEMM tile prefix) inside a workspace that the
// caller allocates.  Some callers cannot allocate device memory where they call the
// layer: a plugin hosted by a framework that owns every device allocation and hands out
// none, an engine whose memory plan is frozen at start-up, or a C program that must not
// call cudaMalloc on its hot path because cudaMalloc can synchronise the device.  For
// them this entry point takes only inputs and outputs and keeps its scratch in a fixed
// array compiled into the library.
//
// The array.  `g_noalloc_scratch` is a file-scope static __device__ array of
// MOE_NOALLOC_SCRATCH_BYTES (4 MiB).  Every GPU that loads the library holds it until the
// process exits.  Host code cannot use the array's name as a device address (on the host
// the name is only a stand-in), so the first call on each device, with that device
// current, asks the runtime for the real address with cudaGetSymbolAddress() and caches
// it; that first call should therefore come before any stream capture.  The cached address
// belongs to the device's primary context: after a cudaDeviceReset() it is stale, and the
// entry point must not be called on that device again in the same process.
//
// Sharing.  All calls on a device share the one array and the array keeps the previous
// call's contents.  Nothing in it needs to start at zero: the count kernel writes every
// per-block count and every rank it later reads, and the scan writes the offsets and the
// tile prefix.  Calls whose kernels overlap on the GPU (two streams, or two host threads)
// race on the array; serialise them.
//
// This file is compiled as part of the library's single translation unit (it is
// included at the end of moe_api.cu) so that it launches the same kernels as moe_permute
// and reports device-side errors through the same error word.

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
void* g_noalloc_addr[kNoallocMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int noalloc_scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" int moe_permute_noalloc(const moe_bf16* x, const int32_t* idx, int T, int d, int E, int k,
                                   int64_t capacity, int32_t* counts_raw, int32_t* counts, int32_t* offsets,
                                   int32_t* dest, int32_t* src_token, moe_bf16* x_perm, moe_stream_t stream) {
    using namespace moe;
    int rc = check_shape(T, d, E, k, 64);
    if (rc != MOE_OK) return rc;
    if (!(x && idx && counts_raw && counts && offsets && dest && src_token && x_perm)) return MOE_ERR_INVALID_ARG;
    if (!(aligned16(x) && aligned16(x_perm) && aligned16(idx) && aligned16(dest))) return MOE_ERR_ALIGN;
    size_t o_blk, o_rank, o_mp;
    const size_t need = permute_scratch_bytes(T, E, k, &o_blk, &o_rank, &o_mp);
    if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;   // beyond the fixed scratch
    DeviceInfo* di;
    if ((rc = device_info(&di)) != MOE_OK) return rc;
    void* scratch = nullptr;
    if ((rc = noalloc_scratch_address(&scratch)) != MOE_OK) return rc;
    char* base = static_cast<char*>(scratch);
    return run_permute(di, x, idx, T, d, E, k, capacity < 0 ? -1 : (long long)capacity, counts_raw, counts, offsets,
                       dest, src_token, x_perm, reinterpret_cast<int32_t*>(base + o_blk),
                       reinterpret_cast<int32_t*>(base + o_rank), reinterpret_cast<int32_t*>(base + o_mp),
                       static_cast<cudaStream_t>(stream));
}
