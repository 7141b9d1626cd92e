// lr_decode.cu -- one decode step of GQA attention over the long-range
// reference encoding (the training-free part of DeltaKV), for sm_100a.
//
// Page "DeltaKV" (gist.science summary of arXiv 2602.08005), section A
// ("Reconstruction": the stored residual plus the mean of the chosen
// references) and section 2 (similar tokens lie far apart).  A token p that is
// not a reference reconstructs as x^_p = mean_{r in R_p} x^_r + delta^_p, with
// delta^_p = (code - 8) d the Q4_0 residual; a reference token is its fp16
// value.  The decode never materialises x^: by linearity
//   q . k^_p   = (1/|R_p|) sum_{r in R_p} (q . k^_r) + q . delta^K_p
//   sum_p w_p v^_p = sum_r W_r v^_r + sum_p w_p delta^V_p,
//   W_r = sum_{p : r in R^V_p} w_p / |R^V_p|  (+ w_p for the reference token p = r s).
// Five launches:
//  1. refdot: q . k^_r for every stored K reference (1/stride of the tokens);
//     refmean: every token's reference part of its score (the mean of its
//     references' dots), written where the split kernel completes the score.
//  2. split: one warp per chunk of a sequence (sized so the grid fills one
//     wave; at least 128 tokens).  Each 32-token tile's
//     codes are staged in shared memory as exact fp16 (code - 8); the K side
//     is an MMA with the tokens as rows (ldmatrix), the scores add the mean of
//     the reference dots; online softmax; the V side is an MMA with the
//     channels as rows (ldmatrix.trans) against the weights times the V
//     scales, each an fp16 hi + lo pair.  The raw scores are kept for step 3,
//     and a partial (max, sum, output) record per chunk.
//  3. combine, in two launches: log-sum-exp over the chunks and the final
//     weight of every token scattered onto its V references (W_r), one block
//     per chunk; then out = the merged delta part + sum_r W_r v^_r, one block
//     per head.
// Inputs are the canonical layouts dkv_lr_encode writes.
#include <atomic>
#include <cstdint>
#include <mutex>

#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace dkv {

constexpr int LRD_TILE = 32;                // tokens per staged tile
constexpr int LRD_CHUNK_MIN = 128;          // tokens per split warp, at least (the host sizes
                                            // chunks so the split grid fills one wave)
constexpr int LRD_WARPS = 4;
constexpr int LRD_ROW = D + 8;              // staged row stride (halves): 272 B, conflict-free
constexpr int LRD_PARTIAL = 8 + 8 + 8 * D;  // m[8], l[8], o[8][128]

struct LrdTensor {
    const int32_t *ref;          // [n_seq][T][m]
    const uint16_t *ref_values;  // [n_seq][NR][D]
    const uint16_t *scales;      // [n_seq][T][4]
    const uint8_t *codes;        // [n_seq][T][D]
};

struct LrdArgs {
    LrdTensor k, v;
    int B, Hkv, T, s, m, Hq, G, NR, n_chunks;
    int chunk;                   // tokens per split warp (a multiple of LRD_TILE)
    const int32_t *lens;         // [B] device
    const void *Q;
    int q_dtype;
    float scale_log2;            // softmax_scale * log2(e)
    float *dots;                 // [n_seq][NR][8]
    float *S;                    // [n_seq][T][8] raw scores (q . k^)
    float *part;                 // [n_seq][n_chunks][LRD_PARTIAL]
    float *W;                    // [n_seq][NR][8]
    float *out;                  // [B][Hq][D]
};

__device__ inline int lrd_len(const LrdArgs &a, int b) {
    const int l = a.lens ? a.lens[b] : a.T;
    return l < 0 ? 0 : (l > a.T ? a.T : l);
}

__device__ inline float lrd_q(const LrdArgs &a, int64_t i) {
    if (a.q_dtype == DKV_F32) return static_cast<const float *>(a.Q)[i];
    if (a.q_dtype == DKV_F16) return __half2float(static_cast<const __half *>(a.Q)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(a.Q)[i]);
}

// ---------------------------------------------------------------------------
// 1. q . k^_r for the references of one sequence: one warp per reference,
//    lanes hold channels 4 lane .. 4 lane + 3, binary32 products in order.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(LRD_WARPS * 32) lrd_refdot_kernel(LrdArgs a) {
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel
    const int seq = blockIdx.y, b = seq / a.Hkv, kvh = seq % a.Hkv;
    const int lane = threadIdx.x & 31;
    const int nr = (lrd_len(a, b) + a.s - 1) / a.s;
    float q[8][4];
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q[h][i] = h < a.G ? lrd_q(a, ((int64_t)b * a.Hq + kvh * a.G + h) * D + 4 * lane + i) : 0.f;
    for (int r = blockIdx.x * LRD_WARPS + (threadIdx.x >> 5); r < nr; r += gridDim.x * LRD_WARPS) {
        const uint2 kv = *reinterpret_cast<const uint2 *>(a.k.ref_values +
                                                          ((int64_t)seq * a.NR + r) * D + 4 * lane);
        const float k0 = h_lo(kv.x), k1 = h_hi(kv.x), k2 = h_lo(kv.y), k3 = h_hi(kv.y);
        float d[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            float x = q[h][0] * k0;
            x = fmaf(q[h][1], k1, x);
            x = fmaf(q[h][2], k2, x);
            x = fmaf(q[h][3], k3, x);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            d[h] = x;
        }
        if (lane < 8) {
            float v = d[0];
#pragma unroll
            for (int h = 1; h < 8; ++h) if (lane == h) v = d[h];
            a.dots[((int64_t)seq * a.NR + r) * 8 + lane] = v;
        }
    }
}

// Stage the codes of tokens [p0, p0 + 32) of one tensor as fp16 (code - 8)
// into `dst` ([32][LRD_ROW] halves); rows past the sequence are zero.
__device__ inline void lrd_stage(const uint8_t *codes, int64_t row0, int p0, int p_end,
                                 __half *dst, int lane) {
    const uint32_t mag = 0x64646464u;       // high bytes of fp16 1024 + n
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int r = it * 4 + (lane >> 3), ci = lane & 7;    // row, 16-byte chunk
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        const bool in = p0 + r < p_end;
        if (in) w = *reinterpret_cast<const uint4 *>(codes + (row0 + p0 + r) * D + 16 * ci);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        uint32_t h[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            h[2 * k] = in ? hsub2_1032(prmt(ww[k], mag, 0x5140u)) : 0u;
            h[2 * k + 1] = in ? hsub2_1032(prmt(ww[k], mag, 0x5342u)) : 0u;
        }
        uint4 *d4 = reinterpret_cast<uint4 *>(dst + r * LRD_ROW + 16 * ci);
        d4[0] = make_uint4(h[0], h[1], h[2], h[3]);
        d4[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
}

// Mean of the reference dots of token p for heads (h0, h0 + 1), or the
// reference's own dot when p is a reference.
__device__ inline float2 lrd_refpart(const LrdArgs &a, int seq, int p, int h0) {
    const int64_t db = (int64_t)seq * a.NR;
    if (p % a.s == 0) {
        return *reinterpret_cast<const float2 *>(a.dots + (db + p / a.s) * 8 + h0);
    }
    const int32_t *rp = a.k.ref + ((int64_t)seq * a.T + p) * a.m;
    float s0 = 0.f, s1 = 0.f;
    int me = 0;
    for (int k = 0; k < a.m; ++k) {
        const int r = rp[k];
        if (r < 0) break;
        const float2 d = *reinterpret_cast<const float2 *>(a.dots + (db + r) * 8 + h0);
        s0 = __fadd_rn(s0, d.x);
        s1 = __fadd_rn(s1, d.y);
        ++me;
    }
    const float inv = me > 0 ? 1.f / (float)me : 0.f;
    return make_float2(s0 * inv, s1 * inv);
}

// 1b. The reference part of every token's score, into S (the split kernel
//     adds the token's own residual dot): one thread per (token, head pair).
__global__ void __launch_bounds__(256) lrd_refmean_kernel(LrdArgs a) {
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel
    const int seq = blockIdx.y, b = seq / a.Hkv;
    const int len = lrd_len(a, b);
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // token * 4 + head pair
    // the sequence's reference weights W_r start at 0 (the combine adds to them)
    for (int64_t k = i; k < (int64_t)a.NR * 8; k += (int64_t)gridDim.x * blockDim.x)
        a.W[(int64_t)seq * a.NR * 8 + k] = 0.f;
    const int p = (int)(i >> 2), hp = (int)(i & 3);
    if (p >= len) return;
    const float2 rp = lrd_refpart(a, seq, p, 2 * hp);
    *reinterpret_cast<float2 *>(a.S + ((int64_t)seq * a.T + p) * 8 + 2 * hp) = rp;
}

// ---------------------------------------------------------------------------
// 2. split: one warp per (sequence, chunk of a.chunk tokens).  QHL: fp32 queries as
//    an fp16 hi + lo pair.
// ---------------------------------------------------------------------------
template <bool QHL>
__global__ void __launch_bounds__(LRD_WARPS * 32) lrd_split_kernel(LrdArgs a) {
    extern __shared__ __align__(128) uint8_t lrd_smem[];
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int64_t item = (int64_t)blockIdx.x * LRD_WARPS + warp;
    if (item >= (int64_t)a.B * a.Hkv * a.n_chunks) return;       // uniform over the warp
    const int seq = (int)(item / a.n_chunks), chunk = (int)(item % a.n_chunks);
    const int b = seq / a.Hkv, kvh = seq % a.Hkv;
    const int len = lrd_len(a, b);
    const int pb = chunk * a.chunk, pe = min(len, pb + a.chunk);
    if (pb >= pe) return;
    __half *Kc = reinterpret_cast<__half *>(lrd_smem) + warp * 2 * LRD_TILE * LRD_ROW;
    __half *Vc = Kc + LRD_TILE * LRD_ROW;
    const int64_t row0 = (int64_t)seq * a.T;

    // q of head gq (n column) as B fragments
    uint32_t qb[8][2], ql[8][2];
    {
        const bool ok = gq < a.G;
        const int64_t qrow = ((int64_t)b * a.Hq + kvh * a.G + (ok ? gq : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c = 16 * kk + 2 * tq;
            const float q0 = ok ? lrd_q(a, qrow + c) : 0.f, q1 = ok ? lrd_q(a, qrow + c + 1) : 0.f;
            const float q8 = ok ? lrd_q(a, qrow + c + 8) : 0.f, q9 = ok ? lrd_q(a, qrow + c + 9) : 0.f;
            qb[kk][0] = h2_as_u32(__floats2half2_rn(q0, q1));
            qb[kk][1] = h2_as_u32(__floats2half2_rn(q8, q9));
            if (QHL) {
                ql[kk][0] = h2_as_u32(__floats2half2_rn(q0 - h_lo(qb[kk][0]), q1 - h_hi(qb[kk][0])));
                ql[kk][1] = h2_as_u32(__floats2half2_rn(q8 - h_lo(qb[kk][1]), q9 - h_hi(qb[kk][1])));
            }
        }
    }
    float m_run[2] = {-1e30f, -1e30f}, l_run[2] = {0.f, 0.f};
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    const bool h_ok0 = 2 * tq < a.G, h_ok1 = 2 * tq + 1 < a.G;

#pragma unroll 1
    for (int p0 = pb; p0 < pe; p0 += LRD_TILE) {
        __syncwarp();
        lrd_stage(a.k.codes, row0, p0, pe, Kc, lane);
        lrd_stage(a.v.codes, row0, p0, pe, Vc, lane);
        __syncwarp();
        // ---- K side: x[mt][r][e], token p0 + 16 mt + g + 8 r, head 2 tq + e
        float x[2][2][2];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float acc[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t af[4];
                ldsm_x4(af, Kc + (16 * mt + (lane & 15)) * LRD_ROW + 16 * kk + 8 * (lane >> 4));
                mma16816(acc[kk >> 1], af[0], af[1], af[2], af[3], qb[kk][0], qb[kk][1]);
                if (QHL) mma16816(acc[kk >> 1], af[0], af[1], af[2], af[3], ql[kk][0], ql[kk][1]);
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int p = p0 + 16 * mt + gq + 8 * r;
                uint2 sc = make_uint2(0u, 0u);
                float2 rp = make_float2(0.f, 0.f);
                if (p < pe) {
                    sc = *reinterpret_cast<const uint2 *>(a.k.scales + (row0 + p) * NB);
                    rp = *reinterpret_cast<const float2 *>(a.S + (row0 + p) * 8 + 2 * tq);
                }
                const float d0 = h_lo(sc.x), d1 = h_hi(sc.x), d2 = h_lo(sc.y), d3 = h_hi(sc.y);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = acc[0][2 * r + e] * d0;
                    v = fmaf(acc[1][2 * r + e], d1, v);
                    v = fmaf(acc[2][2 * r + e], d2, v);
                    v = fmaf(acc[3][2 * r + e], d3, v);
                    x[mt][r][e] = v + (e ? rp.y : rp.x);
                }
                if (p < pe) {
                    float *sp = a.S + (row0 + p) * 8 + 2 * tq;
                    *reinterpret_cast<float2 *>(sp) = make_float2(x[mt][r][0], x[mt][r][1]);
                }
            }
        }
        // ---- online softmax for heads 2 tq + e
        float alpha[2], w[2][2][2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const bool hok = e ? h_ok1 : h_ok0;
            float mx = -INFINITY;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const bool ok = hok && p0 + 16 * mt + gq + 8 * r < pe;
                    x[mt][r][e] = ok ? x[mt][r][e] : -INFINITY;
                    mx = fmaxf(mx, x[mt][r][e]);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run[e], mx * a.scale_log2);
            alpha[e] = exp2f(m_run[e] - m_new);
            m_run[e] = m_new;
            float ps = 0.f;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    w[mt][r][e] = exp2f(fmaf(x[mt][r][e], a.scale_log2, -m_new));
                    ps += w[mt][r][e];
                }
            l_run[e] = l_run[e] * alpha[e] + ps;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o[i][0] *= alpha[0]; o[i][1] *= alpha[1];
            o[i][2] *= alpha[0]; o[i][3] *= alpha[1];
        }
        // ---- V side: o[c][h] += sum_p delta^V_p[c] * w_p[h]; k-tile kt = the
        //      16 tokens of m-tile kt; B = w * dV as an fp16 hi + lo pair
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            uint2 dv[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int p = p0 + 16 * kt + gq + 8 * r;
                dv[r] = p < pe ? *reinterpret_cast<const uint2 *>(a.v.scales + (row0 + p) * NB)
                               : make_uint2(0u, 0u);
            }
            const uint32_t wh0 = pack_h2(w[kt][0][0], w[kt][0][1]);
            const uint32_t wh1 = pack_h2(w[kt][1][0], w[kt][1][1]);
            const uint32_t wl0 = pack_h2(w[kt][0][0] - h_lo(wh0), w[kt][0][1] - h_hi(wh0));
            const uint32_t wl1 = pack_h2(w[kt][1][0] - h_lo(wh1), w[kt][1][1] - h_hi(wh1));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t u0 = (j < 2) ? dv[0].x : dv[0].y, u1 = (j < 2) ? dv[1].x : dv[1].y;
                const __half2 d0 = (j & 1) ? __high2half2(u32_as_h2(u0)) : __low2half2(u32_as_h2(u0));
                const __half2 d1 = (j & 1) ? __high2half2(u32_as_h2(u1)) : __low2half2(u32_as_h2(u1));
                const __half2 h0 = __hmul2(u32_as_h2(wh0), d0), h1 = __hmul2(u32_as_h2(wh1), d1);
                const __half2 l0 = __hfma2(u32_as_h2(wl0), d0, __hfma2(u32_as_h2(wh0), d0, __hneg2(h0)));
                const __half2 l1 = __hfma2(u32_as_h2(wl1), d1, __hfma2(u32_as_h2(wh1), d1, __hneg2(h1)));
                const uint32_t b0 = movm_t(h2_as_u32(h0)), b1 = movm_t(h2_as_u32(h1));
                const uint32_t c0 = movm_t(h2_as_u32(l0)), c1 = movm_t(h2_as_u32(l1));
#pragma unroll
                for (int mh = 0; mh < 2; ++mh) {
                    const int mtc = 2 * j + mh;         // 16-channel m-tile
                    uint32_t af[4];
                    ldsm_x4_t(af, Vc + (16 * kt + (lane & 7) + 8 * (lane >> 4)) * LRD_ROW +
                                      16 * mtc + 8 * ((lane >> 3) & 1));
                    mma16816(o[mtc], af[0], af[1], af[2], af[3], b0, b1);
                    mma16816(o[mtc], af[0], af[1], af[2], af[3], c0, c1);
                }
            }
        }
    }
    // ---- the chunk's partial record
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float l = l_run[e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_run[e] = l;
    }
    float *rec = a.part + ((int64_t)seq * a.n_chunks + chunk) * LRD_PARTIAL;
    if (gq == 0) {
        rec[2 * tq] = m_run[0];
        rec[2 * tq + 1] = m_run[1];
        rec[8 + 2 * tq] = l_run[0];
        rec[8 + 2 * tq + 1] = l_run[1];
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        const int c0 = 16 * mt + gq;
        rec[16 + (2 * tq) * D + c0] = o[mt][0];
        rec[16 + (2 * tq + 1) * D + c0] = o[mt][1];
        rec[16 + (2 * tq) * D + c0 + 8] = o[mt][2];
        rec[16 + (2 * tq + 1) * D + c0 + 8] = o[mt][3];
    }
}

// ---------------------------------------------------------------------------
// 3. combine, in two launches.
//  weights: one block per (chunk, sequence): the log-sum-exp over
//    the sequence's chunks, then the final weight of each of the chunk's
//    tokens added onto its V references (W_r, zeroed by refmean).
//  output: one block per (head, sequence), one thread per channel: the merged
//    delta part plus sum_r W_r v^_r (the head's W_r read once into shared
//    memory when they fit).
// ---------------------------------------------------------------------------
// Log-sum-exp statistics of head h over the nch chunk records of a sequence:
// the largest chunk maximum M and the sum L of the chunk sums rescaled to it.
__device__ inline void lrd_lse(const float *part, int nch, int h, float &M, float &L) {
    M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, part[(int64_t)c * LRD_PARTIAL + h]);
    L = 0.f;
    for (int c = 0; c < nch; ++c)
        L += part[(int64_t)c * LRD_PARTIAL + 8 + h] * exp2f(part[(int64_t)c * LRD_PARTIAL + h] - M);
}

constexpr int LRD_WEIGHT_THREADS = 256;

__global__ void __launch_bounds__(LRD_WEIGHT_THREADS) lrd_weights_kernel(LrdArgs a) {
    __shared__ float Mh[8], Lh[8];
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel
    const int chunk = blockIdx.x, seq = blockIdx.y, b = seq / a.Hkv;
    const int len = lrd_len(a, b);
    const int pb = chunk * a.chunk, pe = min(len, pb + a.chunk);
    if (pb >= pe) return;                                   // uniform over the block
    const int nch = (len + a.chunk - 1) / a.chunk;
    const float *part = a.part + (int64_t)seq * a.n_chunks * LRD_PARTIAL;
    if ((int)threadIdx.x < a.G) lrd_lse(part, nch, threadIdx.x, Mh[threadIdx.x], Lh[threadIdx.x]);
    __syncthreads();
    float *W = a.W + (int64_t)seq * a.NR * 8;
    const int32_t *vref = a.v.ref + (int64_t)seq * a.T * a.m;
    const float *S = a.S + (int64_t)seq * a.T * 8;
    for (int p = pb + threadIdx.x; p < pe; p += blockDim.x) {
        const bool isref = p % a.s == 0;
        int me = 0;
        if (!isref)
            while (me < a.m && vref[(int64_t)p * a.m + me] >= 0) ++me;
        const float inv = isref ? 1.f : 1.f / (float)me;
        for (int h = 0; h < a.G; ++h) {
            const float wv = exp2f(fmaf(S[(int64_t)p * 8 + h], a.scale_log2, -Mh[h])) / Lh[h];
            if (isref) {
                atomicAdd(W + (int64_t)(p / a.s) * 8 + h, wv);
            } else {
                for (int k = 0; k < me; ++k)
                    atomicAdd(W + (int64_t)vref[(int64_t)p * a.m + k] * 8 + h, wv * inv);
            }
        }
    }
}

// The head's W_r in shared memory when NR floats fit in the default 48 KB.
constexpr int LRD_W_SMEM_MAX = 48 * 1024;

template <bool WSM>
__global__ void __launch_bounds__(D) lrd_out_kernel(LrdArgs a) {
    extern __shared__ float w_sm[];                         // WSM: [NR]
    __shared__ float Ms, Ls;
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel
    const int h = blockIdx.x, seq = blockIdx.y, b = seq / a.Hkv, kvh = seq % a.Hkv;
    const int len = lrd_len(a, b), c = threadIdx.x;
    float *out = a.out + ((int64_t)b * a.Hq + kvh * a.G + h) * D;
    if (len == 0) {                                         // uniform over the block
        out[c] = 0.f;
        return;
    }
    const int nch = (len + a.chunk - 1) / a.chunk;
    const int nr = (len + a.s - 1) / a.s;
    const float *part = a.part + (int64_t)seq * a.n_chunks * LRD_PARTIAL;
    if (c == 0) {
        float M, L;
        lrd_lse(part, nch, h, M, L);
        Ms = M;
        Ls = L;
    }
    const float *W = a.W + (int64_t)seq * a.NR * 8;
    if constexpr (WSM)
        for (int r = c; r < nr; r += blockDim.x) w_sm[r] = W[(int64_t)r * 8 + h];
    __syncthreads();
    // out = merged delta part + sum_r W_r v^_r
    float acc = 0.f;
#pragma unroll 4
    for (int ch = 0; ch < nch; ++ch) {
        const float *rec = part + (int64_t)ch * LRD_PARTIAL;
        acc = fmaf(rec[16 + h * D + c], exp2f(rec[h] - Ms), acc);
    }
    acc /= Ls;
    const uint16_t *rv = a.v.ref_values + (int64_t)seq * a.NR * D;
#pragma unroll 8
    for (int r = 0; r < nr; ++r)
        acc = fmaf(WSM ? w_sm[r] : W[(int64_t)r * 8 + h],
                   __half2float(__ushort_as_half(rv[(int64_t)r * D + c])), acc);
    out[c] = acc;
}

size_t lrd_workspace_floats(int B, int Hkv, int T, int s) {
    const int64_t nseq = (int64_t)B * Hkv, NR = (T + s - 1) / s;
    const int64_t nch = (T + LRD_CHUNK_MIN - 1) / LRD_CHUNK_MIN;
    return (size_t)(nseq * NR * 8 * 2 + nseq * (int64_t)T * 8 + nseq * nch * LRD_PARTIAL);
}


// The split kernel's resident warps on the current device (its shared-memory
// attribute is set on the first call), cached per device and query variant.
constexpr size_t kLrdSplitSmem = (size_t)LRD_WARPS * 2 * LRD_TILE * LRD_ROW * sizeof(__half);
constexpr int kLrdMaxDevices = 64;
static std::mutex g_lrd_mu;

static cudaError_t lrd_split_resident(bool qhl, int64_t *resident) {
    static std::atomic<int64_t> res_of[2][kLrdMaxDevices];   // 0: not computed yet
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kLrdMaxDevices) return cudaErrorInvalidDevice;
    int64_t r = res_of[qhl][dev].load(std::memory_order_acquire);
    if (r == 0) {
        std::lock_guard<std::mutex> lock(g_lrd_mu);
        r = res_of[qhl][dev].load(std::memory_order_relaxed);
        if (r == 0) {
            const void *fn = qhl ? (const void *)lrd_split_kernel<true>
                                 : (const void *)lrd_split_kernel<false>;
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kLrdSplitSmem);
            if (e != cudaSuccess) return e;
            int per_sm = 0, nsm = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, LRD_WARPS * 32,
                                                              kLrdSplitSmem);
            if (e != cudaSuccess) return e;
            e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            r = (int64_t)(per_sm < 1 ? 1 : per_sm) * nsm * LRD_WARPS;
            res_of[qhl][dev].store(r, std::memory_order_release);
        }
    }
    *resident = r;
    return cudaSuccess;
}

cudaError_t launch_lr_decode(const LrdView &K, const LrdView &V, int B, int Hkv, int T, int s,
                             int m, const int32_t *lens, const void *Q, int q_dtype, int Hq,
                             float softmax_scale, float *out, float *ws, cudaStream_t st) {
    LrdArgs a;
    a.k = LrdTensor{K.ref, K.ref_values, K.scales, K.codes};
    a.v = LrdTensor{V.ref, V.ref_values, V.scales, V.codes};
    a.B = B; a.Hkv = Hkv; a.T = T; a.s = s; a.m = m; a.Hq = Hq; a.G = Hq / Hkv;
    a.NR = (T + s - 1) / s;
    a.lens = lens; a.Q = Q; a.q_dtype = q_dtype;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    const int64_t nseq = (int64_t)B * Hkv;
    a.dots = ws;
    a.W = a.dots + nseq * a.NR * 8;
    a.S = a.W + nseq * a.NR * 8;
    a.part = a.S + nseq * (int64_t)T * 8;
    a.out = out;
    dim3 g1((unsigned)min(1024, (a.NR + LRD_WARPS - 1) / LRD_WARPS), (unsigned)nseq);
    cudaError_t e = launch_pdl(lrd_refdot_kernel, g1, dim3(LRD_WARPS * 32), 0, st, a);
    if (e != cudaSuccess) return e;
    dim3 g2((unsigned)(((int64_t)T * 4 + 255) / 256), (unsigned)nseq);
    e = launch_pdl(lrd_refmean_kernel, g2, dim3(256), 0, st, a);
    if (e != cudaSuccess) return e;
    // chunks sized so that the split grid fills one wave of resident warps:
    // chunks per sequence = resident warps / sequences, whole 32-token tiles,
    // at least LRD_CHUNK_MIN tokens (the workspace is sized for that)
    const size_t smem = kLrdSplitSmem;
    int64_t resident = 0;
    e = lrd_split_resident(q_dtype == DKV_F32, &resident);
    if (e != cudaSuccess) return e;
    const int64_t per_seq = resident / nseq > 1 ? resident / nseq : 1;
    int64_t chunk = (T + per_seq - 1) / per_seq;
    chunk = (chunk + LRD_TILE - 1) / LRD_TILE * LRD_TILE;
    a.chunk = (int)(chunk < LRD_CHUNK_MIN ? LRD_CHUNK_MIN : chunk);
    a.n_chunks = (T + a.chunk - 1) / a.chunk;
    const int64_t warps = nseq * a.n_chunks;
    const unsigned ctas = (unsigned)((warps + LRD_WARPS - 1) / LRD_WARPS);
    e = q_dtype == DKV_F32
            ? launch_pdl(lrd_split_kernel<true>, dim3(ctas), dim3(LRD_WARPS * 32), smem, st, a)
            : launch_pdl(lrd_split_kernel<false>, dim3(ctas), dim3(LRD_WARPS * 32), smem, st, a);
    if (e != cudaSuccess) return e;
    e = launch_pdl(lrd_weights_kernel, dim3((unsigned)a.n_chunks, (unsigned)nseq),
                   dim3(LRD_WEIGHT_THREADS), 0, st, a);
    if (e != cudaSuccess) return e;
    const size_t wsm = (size_t)a.NR * sizeof(float);
    return wsm <= (size_t)LRD_W_SMEM_MAX
               ? launch_pdl(lrd_out_kernel<true>, dim3((unsigned)a.G, (unsigned)nseq), dim3(D), wsm,
                            st, a)
               : launch_pdl(lrd_out_kernel<false>, dim3((unsigned)a.G, (unsigned)nseq), dim3(D), 0,
                            st, a);
}

}  // namespace dkv
