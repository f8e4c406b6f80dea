// Allocation-free decode entry point.
//
// kvq_decode_attention needs a caller-provided device workspace.  Some
// callers cannot provide one: code that may not call cudaMalloc at all (a
// serving loop with a fixed device-memory budget reserved at start-up, a
// plugin inside a host framework that owns every device allocation, code
// running where the allocator is unavailable or must not be touched).  For
// them, kvq_decode_attention_noalloc runs the very same decode kernels with
// the workspace placed in a fixed array in the library's own device memory.
//
// That array is a file-scope __device__ variable of KVQ_NOALLOC_SCRATCH_BYTES
// bytes: every GPU that loads the library holds it until the process exits.
// Host code cannot use the array's name as a device address, so the first
// call on each device looks the address up once (cudaGetSymbolAddress, with
// that device current) and caches it; that first call should therefore come
// before any stream capture.  The decode kernels need no zeroed workspace,
// so nothing is cleared between calls.  All calls share the one array:
// calls that overlap on the GPU (different streams, or different host
// threads on the same device) race on it and must be serialised by the
// caller.
#include <mutex>

#include "kvq_internal.cuh"

namespace {

constexpr size_t kScratchBytes = KVQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const uint16_t *Q, int32_t Hq,
                                                   const kvq_cache_desc *cache, kvq_rot_mode mode,
                                                   const float *R_k, const float *R_v,
                                                   const int32_t *perm, const int32_t *seq_lens,
                                                   int32_t sink_fp16, int32_t max_ctx,
                                                   uint16_t *out, void *stream) {
    if (!cache) return KVQ_ERR_INVALID_ARG;
    int dev = -1, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return KVQ_ERR_CUDA;
    // the workspace this call needs must fit the fixed array
    const size_t need = kvq_decode_workspace_size(cache->B, Hq, cache->Hkv, max_ctx, sms);
    if (need == 0) return KVQ_ERR_INVALID_ARG;
    if (need > kScratchBytes) return KVQ_ERR_WORKSPACE;
    void *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return KVQ_ERR_CUDA;
    return kvq_decode_attention(Q, Hq, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16, max_ctx,
                                ws, kScratchBytes, out, stream);
}
