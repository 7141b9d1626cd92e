// encode.cu -- quantise K/V into the cache (encode a whole prefix, or append
// new tokens continuing the closed loop), plus the two read-back kernels
// (canonical export for bit-exact comparison, fp32 reconstruction for MSE).
//
// Method (page "영상 압축 기법을 KV 캐시에 적용해 Q4 양자화 오차를 10,000배
// 줄인 Delta-KV", sections "핵심 아이디어" and "벤치마크"): position p of a
// sequence is a keyframe iff p mod kf == 0 and is stored as fp16; every other
// position stores delta = x_p - x^_{p-1} with the Q4_0 block rule, where x^ is
// the reconstruction (closed loop, section "컨텍스트 길이에 따른 안정성").
// Each quantiser step is one IEEE fp32 operation in a fixed order (__fsub_rn,
// __fdiv_rn, __fadd_rn, __fmul_rn), so codes and scales are bit-exact with any
// other implementation that takes the same steps in the same order (m / -8 is
// taken as m * -0.125: the same real value, rounded once, so the same bits).
#include <cstdint>

#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace dkv {

struct EncodeArgs {
    CacheView cv;
    const void *K;
    const void *V;
    int dtype;
    const int32_t *seq_lens;   // encode: per-batch lengths (may be null -> T_in)
    int T_in;                  // positions per sequence in the input arrays
    int append;                // 0: encode from position 0; 1: append at seq_len
};

// Range of positions [start, start + n) that batch entry b encodes, or n < 0
// if the entry is skipped (an error was recorded).
__device__ inline void encode_range(const EncodeArgs &a, int b, int &start, int &n) {
    if (a.append) {
        start = a.cv.seqlen[b];
        n = a.T_in;
        if (start < 0 || start > a.cv.cap) { n = -1; return; }
        if (start + n > a.cv.cap) { n = -2; return; }
    } else {
        start = 0;
        n = a.seq_lens ? a.seq_lens[b] : a.T_in;
        if (n < 0 || n > a.T_in || n > a.cv.cap) { n = -1; return; }
    }
}

// Pointers into the data area for (b, kvh).
__device__ inline uint8_t *seq_base(const CacheView &cv, int b, int kvh) {
    return cv.data + ((int64_t)b * cv.Hkv + kvh) * cv.seq_stride;
}

// Pack the codes of `cnt` positions (smem rows 0..cnt-1, 128 codes each) into
// the permuted nibble layout of tensor t, 64 B per position, at dst.
__device__ inline void pack_nibbles(const uint8_t (*codes)[D], int cnt, int t, uint8_t *dst) {
    for (int idx = threadIdx.x; idx < cnt * 16; idx += blockDim.x) {
        int s = idx >> 4, w = idx & 15;
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) word |= (uint32_t)(codes[s][nib_channel(t, w, i)] & 15) << (4 * i);
        reinterpret_cast<uint32_t *>(dst + (int64_t)s * NIB_BYTES)[w] = word;
    }
}

// Grid: x = work item within the batch entry's range (a group for DELTA, a
// 32-position chunk otherwise), y = kvh * 2 + tensor, z = batch.  128 threads:
// warp j handles channels 32j..32j+31 (one quantisation block).
template <int FMT>
__global__ void __launch_bounds__(128) encode_kernel(EncodeArgs a) {
    __shared__ uint8_t codes[SEG][D];
    __shared__ __half scl[SEG][NB];
    const CacheView &cv = a.cv;
    const int b = blockIdx.z, kvh = blockIdx.y >> 1, t = blockIdx.y & 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = warp * 32 + lane;
    const int parity = cv.header[2] & 1;
    float *state_old = cv.state + ((((int64_t)parity * cv.B + b) * cv.Hkv + kvh) * 2 + t) * D;
    float *state_new = cv.state + ((((int64_t)(parity ^ 1) * cv.B + b) * cv.Hkv + kvh) * 2 + t) * D;

    int start, n;
    encode_range(a, b, start, n);
    bool active = n > 0;
    if (n < 0 && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        set_status(cv.header, n == -2 ? DKV_DEV_CAPACITY : DKV_DEV_BAD_SEQLEN);
    if (n <= 0 && blockIdx.x == 0 && FMT == DKV_FMT_DELTA)
        state_new[c] = a.append ? state_old[c] : 0.0f;  // carry the state over

    const void *src = t == 0 ? a.K : a.V;
    const int64_t in_base = (((int64_t)b * cv.Hkv + kvh) * a.T_in) * D;
    uint8_t *sb = seq_base(cv, b, kvh);

    if (active) {
        if (FMT == DKV_FMT_DELTA) {
            const int kf = cv.kf;
            const int g = start / kf + blockIdx.x;
            const int p0 = max(start, g * kf), p1 = min(start + n, (g + 1) * kf);
            uint8_t *rec = p0 < p1 ? rec_ptr(cv, b, kvh, g) : nullptr;
            if (p0 < p1 && !rec) {
                // bad block-table entry (flagged by rec_ptr): nothing written;
                // the state carries over
                if (p1 == start + n) state_new[c] = (p0 % kf) ? state_old[c] : 0.0f;
            } else if (p0 < p1) {
                uint8_t *sc_base = rec + KF_BYTES;
                uint8_t *nib_base = rec + KF_BYTES + (int64_t)(kf - 1) * SC_BYTES +
                                    (int64_t)t * (kf - 1) * NIB_BYTES;
                float xh = (p0 % kf) ? state_old[c] : 0.0f;
                for (int cb = p0; cb < p1; cb += SEG) {
                    const int ce = min(p1, cb + SEG);
                    // first delta index and count of delta positions in [cb, ce)
                    int first_delta = -1, nd = 0;
                    for (int p = cb; p < ce; ++p) {
                        float x = load_in(src, a.dtype, in_base + (int64_t)(p - start) * D + c);
                        if (p % kf == 0) {
                            __half h = __float2half_rn(x);
                            int idx = t == 0 ? k_half_idx(c) : v_half_idx(c);
                            reinterpret_cast<__half *>(rec + t * 256)[idx] = h;
                            xh = __half2float(h);
                        } else {
                            float delta = __fsub_rn(x, xh);
                            __half d16;
                            int code = quant_lane(delta, &d16);
                            int s = p - cb;
                            codes[s][c] = (uint8_t)code;
                            if (lane == 0) scl[s][warp] = d16;
                            xh = __fadd_rn(xh, __fmul_rn((float)(code - 8), __half2float(d16)));
                            if (first_delta < 0) first_delta = p;
                            ++nd;
                        }
                    }
                    __syncthreads();
                    if (nd > 0) {
                        const int s0 = first_delta - cb;              // smem row of it
                        const int di = first_delta - g * kf - 1;      // delta index
                        pack_nibbles(codes + s0, nd, t, nib_base + (int64_t)di * NIB_BYTES);
                        for (int s = threadIdx.x; s < nd; s += blockDim.x) {
                            const __half *hs = scl[s0 + s];
                            uint2 v;
                            v.x = (uint32_t)__half_as_ushort(hs[0]) |
                                  ((uint32_t)__half_as_ushort(hs[1]) << 16);
                            v.y = (uint32_t)__half_as_ushort(hs[2]) |
                                  ((uint32_t)__half_as_ushort(hs[3]) << 16);
                            *reinterpret_cast<uint2 *>(sc_base + (int64_t)(di + s) * SC_BYTES +
                                                       t * 8) = v;
                        }
                    }
                    __syncthreads();
                }
                if (p1 == start + n) state_new[c] = xh;
            }
        } else {
            // Q4_0 / FP16: positions are independent; item = 32-position chunk.
            const int cb = start + blockIdx.x * SEG;
            const int ce = min(start + n, cb + SEG);
            if (cb < ce) {
                if (FMT == DKV_FMT_Q4_0) {
                    uint8_t *sc_base = sb;
                    uint8_t *nib_base = sb + (int64_t)cv.cap * SC_BYTES +
                                        (int64_t)t * cv.cap * NIB_BYTES;
                    for (int p = cb; p < ce; ++p) {
                        float x = load_in(src, a.dtype, in_base + (int64_t)(p - start) * D + c);
                        __half d16;
                        int code = quant_lane(x, &d16);
                        codes[p - cb][c] = (uint8_t)code;
                        if (lane == 0) scl[p - cb][warp] = d16;
                    }
                    __syncthreads();
                    const int nd = ce - cb;
                    pack_nibbles(codes, nd, t, nib_base + (int64_t)cb * NIB_BYTES);
                    for (int s = threadIdx.x; s < nd; s += blockDim.x) {
                        const __half *hs = scl[s];
                        uint2 v;
                        v.x = (uint32_t)__half_as_ushort(hs[0]) |
                              ((uint32_t)__half_as_ushort(hs[1]) << 16);
                        v.y = (uint32_t)__half_as_ushort(hs[2]) |
                              ((uint32_t)__half_as_ushort(hs[3]) << 16);
                        *reinterpret_cast<uint2 *>(sc_base + (int64_t)(cb + s) * SC_BYTES + t * 8) =
                            v;
                    }
                } else {
                    __half *vals = reinterpret_cast<__half *>(sb + (int64_t)t * cv.cap * 256);
                    const int idx = t == 0 ? k_half_idx(c) : v_half_idx(c);
                    for (int p = cb; p < ce; ++p) {
                        float x = load_in(src, a.dtype, in_base + (int64_t)(p - start) * D + c);
                        vals[(int64_t)p * D + idx] = __float2half_rn(x);
                    }
                }
            }
        }
    }

    // The last block to finish publishes the new lengths and flips the state
    // slot; every block has read seq_len and the old state before it arrives.
    __shared__ int last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned total = gridDim.x * gridDim.y * gridDim.z;
        const unsigned prev = atomicAdd(reinterpret_cast<unsigned *>(cv.header + 1), 1u);
        last = prev == total - 1;
    }
    __syncthreads();
    if (last) {
        __threadfence();
        // one thread per batch entry: each reads and then writes its own seq_len
        for (int bb = threadIdx.x; bb < cv.B; bb += blockDim.x) {
            int s0, nn;
            encode_range(a, bb, s0, nn);
            if (nn >= 0) cv.seqlen[bb] = s0 + nn;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            cv.header[2] ^= 1;
            cv.header[1] = 0;
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------------------
// Delta format.  One warp per (batch entry, kv head, keyframe group) of the
// range being written.  The warp carries the group's eight closed loops side
// by side -- K and V, four 32-channel blocks each, lane = channel within its
// block -- so every step of the sequential loop has eight independent
// quantiser chains in flight; the next position's inputs are loaded while the
// current one is quantised.  The nibble words are gathered in the permuted
// layout with warp shuffles (lanes 0-15 write the K words of a position,
// lanes 16-31 the V words) and the scales by lanes 0 and 1.  The quantiser is
// quant_lane, in the same order of steps as the encode of every other path.
// ---------------------------------------------------------------------------
constexpr int ENC_WARPS = 4;

// Input element (tensor t, channel 32 j + lane) of relative position r.
__device__ inline float enc_in(const EncodeArgs &a, int t, int64_t base, int r, int j, int lane) {
    return load_in(t ? a.V : a.K, a.dtype, base + (int64_t)r * D + 32 * j + lane);
}

#ifndef DKV_ENC_MINB
#define DKV_ENC_MINB 1
#endif
__global__ void __launch_bounds__(ENC_WARPS * 32, DKV_ENC_MINB) encode_delta_kernel(EncodeArgs a, int NG) {
    const CacheView &cv = a.cv;
    const int lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * ENC_WARPS + (threadIdx.x >> 5);
    const int kf = cv.kf;
    if (item < (int64_t)cv.B * cv.Hkv * NG) {
        const int gi = (int)(item % NG);
        const int bh = (int)(item / NG);
        const int b = bh / cv.Hkv, kvh = bh % cv.Hkv;
        int start, n;
        encode_range(a, b, start, n);
        const int parity = cv.header[2] & 1;
        const int64_t slot = (int64_t)cv.B * cv.Hkv * 2 * D;
        const int64_t sb = ((int64_t)b * cv.Hkv + kvh) * 2 * D;
        const float *st_old = cv.state + parity * slot + sb;
        float *st_new = cv.state + (parity ^ 1) * slot + sb;
        if (n < 0 && gi == 0 && kvh == 0 && lane == 0)
            set_status(cv.header, n == -2 ? DKV_DEV_CAPACITY : DKV_DEV_BAD_SEQLEN);
        if (n <= 0) {
            if (gi == 0) {                    // nothing written: carry the state over
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int c = t * D + 32 * j + lane;
                        st_new[c] = a.append ? st_old[c] : 0.0f;
                    }
            }
        } else {
            const int g = start / kf + gi;
            const int p0 = max(start, g * kf), p1 = min(start + n, (g + 1) * kf);
            const bool last = p1 == start + n;
            uint8_t *rec = p0 < p1 ? rec_ptr(cv, b, kvh, g) : nullptr;
            if (p0 < p1 && !rec) {
                // bad block-table entry (flagged by rec_ptr): nothing written
                if (last) {
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int c = t * D + 32 * j + lane;
                            st_new[c] = (p0 % kf) ? st_old[c] : 0.0f;
                        }
                }
            } else if (p0 < p1) {
                const int64_t base = ((int64_t)b * cv.Hkv + kvh) * a.T_in * D;
                float xh[2][4], x[2][4];
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        xh[t][j] = (p0 % kf) ? st_old[t * D + 32 * j + lane] : 0.0f;
                        x[t][j] = enc_in(a, t, base, p0 - start, j, lane);
                    }
                const int wt = lane >> 4, ww = lane & 15;   // this lane's nibble word
                uint8_t *nib0 = rec + KF_BYTES + (int64_t)(kf - 1) * SC_BYTES +
                                (int64_t)wt * (kf - 1) * NIB_BYTES + 4 * ww;
#pragma unroll 1
                for (int p = p0; p < p1; ++p) {
                    float xn[2][4];
                    if (p + 1 < p1) {
#pragma unroll
                        for (int t = 0; t < 2; ++t)
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                xn[t][j] = enc_in(a, t, base, p + 1 - start, j, lane);
                    }
                    const int di = p - g * kf;      // 0: keyframe; else delta di - 1
                    if (di == 0) {
#pragma unroll
                        for (int t = 0; t < 2; ++t)
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const __half h = __float2half_rn(x[t][j]);
                                xh[t][j] = __half2float(h);
                                const int ch = 32 * j + lane;
                                reinterpret_cast<__half *>(rec + t * 256)[t == 0 ? k_half_idx(ch)
                                                                                 : v_half_idx(ch)] = h;
                            }
                    } else {
                        uint32_t codes = 0;         // code of (t, j) at bit 16 t + 4 j
                        float dl[8];
                        int cd[8];
                        __half h16[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) dl[i] = __fsub_rn(x[i >> 2][i & 3], xh[i >> 2][i & 3]);
                        quant_lanes<8>(dl, cd, h16);
                        __half d16[2][4];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int t = i >> 2, j = i & 3;
                            d16[t][j] = h16[i];
                            codes |= (uint32_t)cd[i] << (16 * t + 4 * j);
                            xh[t][j] = __fadd_rn(xh[t][j], __fmul_rn((float)(cd[i] - 8),
                                                                     __half2float(h16[i])));
                        }
                        uint32_t word = 0;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int ch = nib_channel(wt, ww, k);
                            const uint32_t v = __shfl_sync(0xffffffffu, codes, ch & 31);
                            word |= ((v >> (16 * wt + 4 * (ch >> 5))) & 15u) << (4 * k);
                        }
                        *reinterpret_cast<uint32_t *>(nib0 + (int64_t)(di - 1) * NIB_BYTES) = word;
                        if (lane < 2) {
                            uint32_t h[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                h[j] = __half_as_ushort(lane ? d16[1][j] : d16[0][j]);
                            *reinterpret_cast<uint2 *>(rec + KF_BYTES + (int64_t)(di - 1) * SC_BYTES +
                                                       lane * 8) =
                                make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
                        }
                    }
                    if (p + 1 < p1) {
#pragma unroll
                        for (int t = 0; t < 2; ++t)
#pragma unroll
                            for (int j = 0; j < 4; ++j) x[t][j] = xn[t][j];
                    }
                }
                if (last) {
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int j = 0; j < 4; ++j) st_new[t * D + 32 * j + lane] = xh[t][j];
                }
            }
        }
    }

    // The last block to finish publishes the new lengths and flips the state
    // slot; every block has read seq_len and the old state before it arrives.
    __shared__ int last_blk;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(reinterpret_cast<unsigned *>(cv.header + 1), 1u);
        last_blk = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (last_blk) {
        __threadfence();
        for (int bb = threadIdx.x; bb < cv.B; bb += blockDim.x) {
            int s0, nn;
            encode_range(a, bb, s0, nn);
            if (nn >= 0) cv.seqlen[bb] = s0 + nn;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            cv.header[2] ^= 1;
            cv.header[1] = 0;
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------------------
// Read-back kernels.  Grid: x = position chunk of 32, y = kvh*2 + t, z = b.
// ---------------------------------------------------------------------------
struct ExportArgs {
    CacheView cv;
    uint8_t *codes;
    uint16_t *scales;
    uint16_t *keyframes;
    float *state;
    float *xhat;        // dequantize target (null for export)
};

template <int FMT>
__global__ void __launch_bounds__(128) readback_kernel(ExportArgs a) {
    const CacheView &cv = a.cv;
    const int b = blockIdx.z, kvh = blockIdx.y >> 1, t = blockIdx.y & 1;
    const int c = threadIdx.x;
    int len = cv.seqlen[b];
    if (len < 0 || len > cv.cap) len = 0;
    const uint8_t *sb = seq_base(cv, b, kvh);
    const int64_t row0 = (((int64_t)b * cv.Hkv + kvh) * 2 + t) * cv.cap;   // [..][cap]
    int nb_, sh;
    if (t == 0) k_nib_pos(c, nb_, sh); else v_nib_pos(c, nb_, sh);
    const int hidx = t == 0 ? k_half_idx(c) : v_half_idx(c);

    if (FMT == DKV_FMT_DELTA) {
        const int kf = cv.kf;
        const int g = blockIdx.x;   // one group per block
        if (g == 0 && a.state) {
            const int parity = cv.header[2] & 1;
            a.state[(((int64_t)b * cv.Hkv + kvh) * 2 + t) * D + c] =
                cv.state[((((int64_t)parity * cv.B + b) * cv.Hkv + kvh) * 2 + t) * D + c];
        }
        if (g * kf >= len) return;
        const uint8_t *rec = rec_ptr(cv, b, kvh, g);
        if (!rec) return;
        const uint8_t *scb = rec + KF_BYTES;
        const uint8_t *nib = rec + KF_BYTES + (int64_t)(kf - 1) * SC_BYTES +
                             (int64_t)t * (kf - 1) * NIB_BYTES;
        const __half kfv = reinterpret_cast<const __half *>(rec + t * 256)[hidx];
        if (a.keyframes)
            a.keyframes[((((int64_t)b * cv.Hkv + kvh) * 2 + t) * cv.n_groups + g) * D + c] =
                __half_as_ushort(kfv);
        float xh = __half2float(kfv);
        const int p1 = min(len, (g + 1) * kf);
        for (int p = g * kf; p < p1; ++p) {
            if (p > g * kf) {
                const int di = p - g * kf - 1;
                const int code = (nib[(int64_t)di * NIB_BYTES + nb_] >> sh) & 15;
                const __half d16 =
                    reinterpret_cast<const __half *>(scb + (int64_t)di * SC_BYTES + t * 8)[c >> 5];
                xh = __fadd_rn(xh, __fmul_rn((float)(code - 8), __half2float(d16)));
                if (a.codes) a.codes[(row0 + p) * D + c] = (uint8_t)code;
                if (a.scales && (c & 31) == 0)
                    a.scales[(row0 + p) * NB + (c >> 5)] = __half_as_ushort(d16);
            } else {
                if (a.codes) a.codes[(row0 + p) * D + c] = 0;
                if (a.scales && (c & 31) == 0) a.scales[(row0 + p) * NB + (c >> 5)] = 0;
            }
            if (a.xhat) a.xhat[(row0 + p) * D + c] = xh;
        }
    } else {
        const int p0 = blockIdx.x * SEG, p1 = min(len, p0 + SEG);
        for (int p = p0; p < p1; ++p) {
            if (FMT == DKV_FMT_Q4_0) {
                const uint8_t *nib = sb + (int64_t)cv.cap * SC_BYTES + (int64_t)t * cv.cap * NIB_BYTES;
                const int code = (nib[(int64_t)p * NIB_BYTES + nb_] >> sh) & 15;
                const __half d16 =
                    reinterpret_cast<const __half *>(sb + (int64_t)p * SC_BYTES + t * 8)[c >> 5];
                if (a.codes) a.codes[(row0 + p) * D + c] = (uint8_t)code;
                if (a.scales && (c & 31) == 0)
                    a.scales[(row0 + p) * NB + (c >> 5)] = __half_as_ushort(d16);
                if (a.xhat) a.xhat[(row0 + p) * D + c] = __fmul_rn((float)(code - 8), __half2float(d16));
            } else {
                const __half v = reinterpret_cast<const __half *>(sb + (int64_t)t * cv.cap * 256 +
                                                                  (int64_t)p * 256)[hidx];
                if (a.keyframes) a.keyframes[(row0 + p) * D + c] = __half_as_ushort(v);
                if (a.xhat) a.xhat[(row0 + p) * D + c] = __half2float(v);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_encode(const CacheView &cv, const void *K, const void *V, int dtype,
                          const int32_t *seq_lens, int T_in, int append, cudaStream_t st) {
    EncodeArgs a{cv, K, V, dtype, seq_lens, T_in, append};
    if (cv.fmt == DKV_FMT_DELTA) {
        // groups a batch entry's range can touch (an append may start mid-group)
        const int NG = (T_in + cv.kf - 1) / cv.kf + (append ? 1 : 0);
        const int64_t warps = (int64_t)cv.B * cv.Hkv * NG;
        const int64_t ctas = (warps + ENC_WARPS - 1) / ENC_WARPS;
        if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
        encode_delta_kernel<<<(unsigned)ctas, ENC_WARPS * 32, 0, st>>>(a, NG);
        return cudaGetLastError();
    }
    int items;
    if (cv.fmt == DKV_FMT_DELTA)
        items = append ? (T_in + cv.kf - 1) / cv.kf + 1 : (T_in + cv.kf - 1) / cv.kf;
    else
        items = (T_in + SEG - 1) / SEG;
    items = items < 1 ? 1 : items;
    dim3 grid(items, cv.Hkv * 2, cv.B);
    switch (cv.fmt) {
        case DKV_FMT_DELTA: encode_kernel<DKV_FMT_DELTA><<<grid, 128, 0, st>>>(a); break;
        case DKV_FMT_Q4_0: encode_kernel<DKV_FMT_Q4_0><<<grid, 128, 0, st>>>(a); break;
        default: encode_kernel<DKV_FMT_FP16><<<grid, 128, 0, st>>>(a); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_readback(const CacheView &cv, uint8_t *codes, uint16_t *scales,
                            uint16_t *keyframes, float *state, float *xhat, cudaStream_t st) {
    ExportArgs a{cv, codes, scales, keyframes, state, xhat};
    int items = cv.fmt == DKV_FMT_DELTA ? cv.n_groups : (cv.cap + SEG - 1) / SEG;
    dim3 grid(items, cv.Hkv * 2, cv.B);
    switch (cv.fmt) {
        case DKV_FMT_DELTA: readback_kernel<DKV_FMT_DELTA><<<grid, 128, 0, st>>>(a); break;
        case DKV_FMT_Q4_0: readback_kernel<DKV_FMT_Q4_0><<<grid, 128, 0, st>>>(a); break;
        default: readback_kernel<DKV_FMT_FP16><<<grid, 128, 0, st>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace dkv
