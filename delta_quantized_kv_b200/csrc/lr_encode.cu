// lr_encode.cu -- long-range reference encoding (the training-free part of
// DeltaKV), for sm_100a.
//
// Page "DeltaKV" (gist.science summary of arXiv 2602.08005): similar tokens lie
// far apart in the context (section 2, long-range inter-token similarity);
// the reference set is the tokens at a fixed stride, a token stores its
// residual against the mean of its most similar references, and the
// reconstruction adds that mean back (section A: Strided Reference Selection,
// Residual Encoding, Reconstruction); the residuals sit near zero and take
// 4-bit quantisation (section 4, 양자화 친화성).  The learned compressor is
// replaced by the Q4_0 block rule.
//
// The steps, in the order both this kernel and any other statement of them
// take them: references are the positions p mod s == 0, stored as fp16; a
// token p chooses among the references r < p the m with the smallest squared
// Euclidean distance to the stored reference (binary64, channels in order,
// each difference, square and sum one IEEE binary64 operation; ties to the
// smaller position); their mean is the binary32 sum in ascending position
// divided by their count; the residual x - mean is quantised with the Q4_0
// block rule and x^ = mean + (code - 8) d.  Every step is one IEEE operation
// in that order, so the choices, codes and scales are bit-exact.
//
// One warp per token; lanes hold channels 32 j + lane.  Each lane ranks the
// candidates g = lane, lane + 32, ... (a sorted list of its m best), and the
// warp merges the lists m times (a butterfly minimum on (distance, position)).
#include <cstdint>

#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace dkv {

constexpr int LR_MAX_M = 8;
constexpr int LR_WARPS = 4;

struct LrArgs {
    const void *X;
    int dtype;
    int n_seq, T, s, m;
    int32_t *ref;
    uint16_t *kfr;
    uint16_t *scales;
    uint8_t *codes;
    float *xhat;
};

// The stored (fp16) value of input element i, as binary32.
__device__ inline float lr_stored(const LrArgs &a, int64_t i) {
    return __half2float(__float2half_rn(load_in(a.X, a.dtype, i)));
}

// (d, g) < (d2, g2): smaller distance, then smaller position.
__device__ inline bool lr_less(double d, int g, double d2, int g2) {
    return d < d2 || (d == d2 && g < g2);
}

__global__ void __launch_bounds__(LR_WARPS * 32) lr_encode_kernel(LrArgs a) {
    __shared__ float xs[LR_WARPS][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.y;
    const int p = blockIdx.x * LR_WARPS + warp;
    if (p >= a.T) return;                // uniform over the warp
    const int s = a.s, m = a.m, T = a.T;
    const int64_t row = (int64_t)seq * T + p;
    const int ng = (T + s - 1) / s;
    float x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[j] = load_in(a.X, a.dtype, row * D + 32 * j + lane);
        xs[warp][32 * j + lane] = x[j];
    }
    __syncwarp();
    if (lane < m) a.ref[row * m + lane] = -1;
    uint8_t *crow = a.codes + row * D;
    if (lane < 4) a.scales[row * (D / 32) + lane] = 0;
    if (p % s == 0) {                    // a reference token: fp16
        const int64_t krow = ((int64_t)seq * ng + p / s) * D;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half h = __float2half_rn(x[j]);
            a.kfr[krow + 32 * j + lane] = __half_as_ushort(h);
            crow[32 * j + lane] = 0;
            if (a.xhat) a.xhat[row * D + 32 * j + lane] = __half2float(h);
        }
        return;
    }
    // rank this lane's candidates: references g = lane, lane + 32, ... below p
    const int nc = (p - 1) / s + 1;
    double bd[LR_MAX_M];
    int bg[LR_MAX_M];
#pragma unroll
    for (int k = 0; k < LR_MAX_M; ++k) { bd[k] = INFINITY; bg[k] = 0x7fffffff; }
    for (int g = lane; g < nc; g += 32) {
        const int64_t rrow = ((int64_t)seq * T + (int64_t)g * s) * D;
        double acc = 0.0;
        for (int c = 0; c < D; ++c) {
            const double diff = __dsub_rn((double)xs[warp][c], (double)lr_stored(a, rrow + c));
            acc = __dadd_rn(acc, __dmul_rn(diff, diff));
        }
        // insert into the sorted list (candidates come in increasing g, so an
        // equal distance stays behind the earlier one)
        if (lr_less(acc, g, bd[LR_MAX_M - 1], bg[LR_MAX_M - 1])) {
            double cd = acc;
            int cg = g;
#pragma unroll
            for (int k = 0; k < LR_MAX_M; ++k) {
                if (lr_less(cd, cg, bd[k], bg[k])) {
                    const double td = bd[k];
                    const int tg = bg[k];
                    bd[k] = cd; bg[k] = cg;
                    cd = td; cg = tg;
                }
            }
        }
    }
    // merge: m times the warp's smallest head
    const int me = min(m, nc);
    int sel[LR_MAX_M];
#pragma unroll
    for (int k = 0; k < LR_MAX_M; ++k) sel[k] = 0x7fffffff;
    for (int k = 0; k < me; ++k) {
        double d = bd[0];
        int g = bg[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double d2 = __shfl_xor_sync(0xffffffffu, d, o);
            const int g2 = __shfl_xor_sync(0xffffffffu, g, o);
            if (lr_less(d2, g2, d, g)) { d = d2; g = g2; }
        }
        sel[k] = g;
        if (bg[0] == g) {                // the owner pops its head
#pragma unroll
            for (int q = 0; q + 1 < LR_MAX_M; ++q) { bd[q] = bd[q + 1]; bg[q] = bg[q + 1]; }
            bd[LR_MAX_M - 1] = INFINITY;
            bg[LR_MAX_M - 1] = 0x7fffffff;
        }
    }
    // ascending position
    for (int i = 1; i < me; ++i)
        for (int j = i; j > 0 && sel[j - 1] > sel[j]; --j) {
            const int t = sel[j]; sel[j] = sel[j - 1]; sel[j - 1] = t;
        }
    if (lane < me) {
        int v = sel[0];
        for (int k = 1; k < me; ++k) if (k == lane) v = sel[k];
        a.ref[row * m + lane] = v;
    }
    // the mean of the chosen references, the residual, the block rule
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = 32 * j + lane;
        float acc = 0.0f;
        for (int k = 0; k < me; ++k)
            acc = __fadd_rn(acc, lr_stored(a, ((int64_t)seq * T + (int64_t)sel[k] * s) * D + c));
        const float mean = __fdiv_rn(acc, (float)me);
        __half d16;
        const int code = quant_lane(__fsub_rn(x[j], mean), &d16);
        crow[c] = (uint8_t)code;
        if (lane == 0) a.scales[row * (D / 32) + j] = __half_as_ushort(d16);
        if (a.xhat)
            a.xhat[row * D + c] =
                __fadd_rn(mean, __fmul_rn((float)(code - 8), __half2float(d16)));
    }
}

cudaError_t launch_lr_encode(const void *X, int dtype, int n_seq, int T, int s, int m,
                             int32_t *ref, uint16_t *kfr, uint16_t *scales, uint8_t *codes,
                             float *xhat, cudaStream_t st) {
    LrArgs a{X, dtype, n_seq, T, s, m, ref, kfr, scales, codes, xhat};
    dim3 grid((T + LR_WARPS - 1) / LR_WARPS, n_seq);
    lr_encode_kernel<<<grid, LR_WARPS * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dkv
