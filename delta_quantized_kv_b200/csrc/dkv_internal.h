// dkv_internal.h -- host-side launchers shared between the C-ABI layer and the
// kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/dkv.h"

namespace dkv {

// The host-side checks every entry point runs on a cache view before any
// launch: DKV_OK, or the status those entry points return for it.
dkv_status validate_cache(const dkv_cache *c);

struct CacheView;

cudaError_t launch_encode(const CacheView &cv, const void *K, const void *V, int dtype,
                          const int32_t *seq_lens, int T_in, int append, cudaStream_t st);
cudaError_t launch_division_check(const float *u, int n, unsigned long long *bad,
                                  cudaStream_t st);
cudaError_t launch_readback(const CacheView &cv, uint8_t *codes, uint16_t *scales,
                            uint16_t *keyframes, float *state, float *xhat, cudaStream_t st);

// Persistent-grid geometry of the split kernel for a cache format on the
// current device: CTAs and warps per CTA.
struct SplitGeom {
    int ctas;
    int warps_per_cta;
};
cudaError_t split_geometry(int fmt, int kf, int64_t max_units, SplitGeom *g);
// Units (keyframe groups, kf > 32: 32-position segments, or 32-position
// chunks) of every sequence of a cache at capacity; nhg = head groups of 8
// virtual heads per kv head.
int64_t split_max_units(int fmt, int kf, int B, int Hkv, int nhg, int cap);

// Floats per partial record: m[8], l[8], o[8][128].
constexpr int PARTIAL_FLOATS = 8 + 8 + 8 * 128;
// Floats per state handed from warp to warp inside a keyframe group (kf > 32):
// the scaled query-key dot of 8 heads and one reconstructed value row.
constexpr int HANDOFF_FLOATS = 8 + 128;
constexpr int HAND_HDR = 4;    // floats before the handoffs: the log2 softmax scale, padding

// nq queries per sequence: query t attends to the positions before
// seq_len - (nq - 1 - t); Q and out are [B][nq][Hq][D].  With cv.len_add = n
// > 0 (delta format) the split kernel first appends the n new tokens K_new,
// V_new ([B][Hkv][n][D] of kv_dtype) and the merge publishes the new lengths.
cudaError_t launch_split(const CacheView &cv, const void *Q, int q_dtype, int Hq, int nq,
                         float softmax_scale, float *ws, int64_t ws_floats, int fault,
                         cudaStream_t st, const void *K_new = nullptr,
                         const void *V_new = nullptr, int kv_dtype = 0);
cudaError_t launch_merge(const CacheView &cv, int Hq, int nq, float *out, const float *ws,
                         int64_t ws_floats, cudaStream_t st);

// Long-range reference encoding of n_seq sequences [n_seq][T][D] (layouts
// of dkv_lr_encode).
cudaError_t launch_lr_encode(const void *X, int dtype, int n_seq, int T, int s, int m,
                             int32_t *ref, uint16_t *kfr, uint16_t *scales, uint8_t *codes,
                             float *xhat, cudaStream_t st);

// Decode over the long-range reference encoding (canonical layouts of
// dkv_lr_encode, one view per tensor); ws holds lrd_workspace_floats floats.
struct LrdView {
    const int32_t *ref;
    const uint16_t *ref_values;
    const uint16_t *scales;
    const uint8_t *codes;
};
size_t lrd_workspace_floats(int B, int Hkv, int T, int s);
cudaError_t launch_lr_decode(const LrdView &K, const LrdView &V, int B, int Hkv, int T, int s,
                             int m, const int32_t *lens, const void *Q, int q_dtype, int Hq,
                             float softmax_scale, float *out, float *ws, cudaStream_t st);

}  // namespace dkv
