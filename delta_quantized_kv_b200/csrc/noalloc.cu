// noalloc.cu -- dkv_decode_attn_noalloc: the decode step without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory at the time they decode: code
// running while a CUDA graph is being captured (cudaMalloc is not allowed
// there), plugins inside a host engine that owns every device allocation and
// plans its memory up front, and latency-critical paths where cudaMalloc's
// implicit device synchronisation is unacceptable.  For them the split
// kernel's partial records live in a fixed array in this library's own device
// memory instead of a workspace the caller passes in.
//
// The array is a file-scope __device__ variable of DKV_NOALLOC_SCRATCH_BYTES
// (16 MiB).  Every GPU that loads the library holds it until the process
// exits.  Its device address is looked up once per device, on the first call
// made with that device current (cudaGetSymbolAddress); make that first call
// before any stream capture.  All calls share the array and it keeps the last
// call's contents; the split kernel writes every record the merge kernel reads
// in the same call, so nothing needs clearing, but two calls that overlap on
// the GPU (different streams, or different caches at the same time) race on
// it and must be serialised by the caller.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/dkv.h"
#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace {

constexpr size_t kScratchFloats = DKV_NOALLOC_SCRATCH_BYTES / sizeof(float);

static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(float **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = static_cast<float *>(p);
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" dkv_status dkv_decode_attn_noalloc(const dkv_cache *cache, const void *Q,
                                              int32_t q_dtype, int32_t n_q_heads,
                                              float softmax_scale, float *out, void *stream) {
    if (!cache || !Q || !out) return DKV_EINVAL;
    const size_t need = dkv_decode_workspace_bytes(&cache->desc, n_q_heads);
    if (need == 0) {
        // invalid descriptor / head count, or no usable device
        if (cache->desc.n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % cache->desc.n_kv_heads)
            return DKV_EINVAL;
        return DKV_ECUDA;
    }
    if (need > DKV_NOALLOC_SCRATCH_BYTES) return DKV_ECAPACITY;
    float *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return DKV_ECUDA;
    return dkv_decode_attn(cache, Q, q_dtype, n_q_heads, softmax_scale, out, ws, need, stream);
}
