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
// exits.  Its device address is looked up (cudaGetSymbolAddress) on the first
// call made with that device current, and again only if the device's context
// has changed since (after cudaDeviceReset the module is loaded anew and the
// array may sit elsewhere); make the first call before any stream capture.
// All calls share the array and it keeps the last call's contents; the split
// kernel writes every record the merge kernel reads in the same call, so
// nothing needs clearing, but two calls that overlap on the GPU (different
// streams, or different caches at the same time) race on it and must be
// serialised by the caller.
#include <cuda.h>            // driver types only: the two driver calls are fetched at run time
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

struct ScratchEntry {
    float *addr;                 // device address of the array (null: not looked up)
    bool have_ctx;               // ctx_id identifies the context addr belongs to
    unsigned long long ctx_id;
};
std::mutex g_mu;
ScratchEntry g_entry[kMaxDevices] = {};

using PfnCtxGetCurrent = CUresult (*)(CUcontext *);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context; false when no context is
// current or the driver does not offer the calls.
bool current_context_id(unsigned long long *id) {
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {                       // under g_mu
        void *a = nullptr, *b = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault) == cudaSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault) == cudaSuccess) {
            get_current = reinterpret_cast<PfnCtxGetCurrent>(a);
            get_id = reinterpret_cast<PfnCtxGetId>(b);
        }
        resolved = true;
    }
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device.
cudaError_t scratch_address(float **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    ScratchEntry &en = g_entry[dev];
    unsigned long long id = 0;
    const bool have = current_context_id(&id);
    if (!en.addr || !have || !en.have_ctx || en.ctx_id != id) {
        void *p = nullptr;
        // (also makes the device's primary context current if none is)
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        en.addr = static_cast<float *>(p);
        en.have_ctx = current_context_id(&en.ctx_id);
    }
    *out = en.addr;
    return cudaSuccess;
}

}  // namespace

extern "C" dkv_status dkv_decode_attn_noalloc(const dkv_cache *cache, const void *Q,
                                              int32_t q_dtype, int32_t n_q_heads,
                                              float softmax_scale, float *out, void *stream) {
    if (!cache || !Q || !out) return DKV_EINVAL;
    // the cache first, with the statuses every other entry point gives it
    const dkv_status s = dkv::validate_cache(cache);
    if (s != DKV_OK) return s;
    if (n_q_heads < 1 || n_q_heads % cache->desc.n_kv_heads != 0) return DKV_EINVAL;
    const size_t need = dkv_decode_workspace_bytes(&cache->desc, n_q_heads);
    if (need == 0) return DKV_ECUDA;        // the device query behind the size failed
    if (need > DKV_NOALLOC_SCRATCH_BYTES) return DKV_ECAPACITY;
    float *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return DKV_ECUDA;
    return dkv_decode_attn(cache, Q, q_dtype, n_q_heads, softmax_scale, out, ws, need, stream);
}
