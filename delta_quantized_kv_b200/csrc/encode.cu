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
// warp j handles channels 32j..32j+31 (one quantisation block).  For the
// delta format this is the variant with the most threads per step (a warp per
// block): it serves appends of a few tokens, where the one-lane-per-block
// kernel below would leave most of the GPU idle.
template <int FMT>
__global__ void __launch_bounds__(128) encode_kernel(EncodeArgs a) {
    __shared__ uint8_t codes[SEG][D];
    __shared__ __half scl[SEG][NB];
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel
    const CacheView &cv = a.cv;
    const int b = blockIdx.z, kvh = blockIdx.y >> 1, t = blockIdx.y & 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = warp * 32 + lane;
    const void *src = t == 0 ? a.K : a.V;
    const int64_t in_base = (((int64_t)b * cv.Hkv + kvh) * a.T_in) * D;
    // An append of a few tokens is latency-bound.  The first input row and
    // both state slots do not depend on the length or on the slot parity, so
    // they are loaded together with those (all in bounds by construction: b,
    // kvh and t index their arrays, and an append has T_in >= 1).
    constexpr bool PF = FMT == DKV_FMT_DELTA && !DKV_CHECKED;
    const int64_t slot = (((int64_t)b * cv.Hkv + kvh) * 2 + t) * D + c;
    const int64_t slot_stride = (int64_t)cv.B * cv.Hkv * 2 * D;
    float x_first = 0.f, st_pf[2] = {0.f, 0.f};
    if (PF && a.append) {
        x_first = load_in(src, a.dtype, in_base + c);
        st_pf[0] = cv.state[slot];
        st_pf[1] = cv.state[slot + slot_stride];
    }
    const int parity = cv.header[2] & 1;
    float *state_old = cv.state + ((((int64_t)parity * cv.B + b) * cv.Hkv + kvh) * 2 + t) * D;
    float *state_new = cv.state + ((((int64_t)(parity ^ 1) * cv.B + b) * cv.Hkv + kvh) * 2 + t) * D;
    const float st_old = (PF && a.append) ? st_pf[parity] : 0.f;   // state_old[c] when PF

    int start, n;
    encode_range(a, b, start, n);
    bool active = n > 0;
    if (n < 0 && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        set_status(cv.header, n == -2 ? DKV_DEV_CAPACITY : DKV_DEV_BAD_SEQLEN);
    if (n <= 0 && blockIdx.x == 0 && FMT == DKV_FMT_DELTA)
        state_new[c] = a.append ? (PF ? st_old : state_old[c]) : 0.0f;  // carry the state over

    uint8_t *sb = seq_base(cv, b, kvh);
    // checked build (block-uniform): this sequence's state rows, its n input
    // rows and, for the comparators, its data
    if (DKV_CHECKED && active) {
        const int es = a.dtype == DKV_F32 ? 4 : 2;
        const int64_t in_bytes = (int64_t)cv.B * cv.Hkv * a.T_in * D * es;
        active = state_ok(cv, state_old, D) && state_ok(cv, state_new, D) &&
                 range_ok(cv.header, static_cast<const uint8_t *>(src) + in_base * es,
                          (int64_t)n * D * es, src, in_bytes) &&
                 (FMT == DKV_FMT_DELTA || rec_ok(cv, sb, cv.seq_stride));
    }

    if (active) {
        if (FMT == DKV_FMT_DELTA) {
            const int kf = cv.kf;
            const int g = start / kf + blockIdx.x;
            const int p0 = max(start, g * kf), p1 = min(start + n, (g + 1) * kf);
            uint8_t *rec = p0 < p1 ? rec_ptr(cv, b, kvh, g) : nullptr;
            if (rec && !rec_ok(cv, rec, cv.rec_bytes)) rec = nullptr;   // checked build
            if (p0 < p1 && !rec) {
                // bad block-table entry (flagged by rec_ptr): nothing written;
                // the state carries over
                if (p1 == start + n)
                    state_new[c] = (p0 % kf) ? ((PF && a.append) ? st_old : state_old[c]) : 0.0f;
            } else if (p0 < p1) {
                uint8_t *sc_base = rec + KF_BYTES;
                uint8_t *nib_base = rec + KF_BYTES + (int64_t)(kf - 1) * SC_BYTES +
                                    (int64_t)t * (kf - 1) * NIB_BYTES;
                float xh = (p0 % kf) ? ((PF && a.append) ? st_old : state_old[c]) : 0.0f;
                for (int cb = p0; cb < p1; cb += SEG) {
                    const int ce = min(p1, cb + SEG);
                    // first delta index and count of delta positions in [cb, ce)
                    int first_delta = -1, nd = 0;
                    for (int p = cb; p < ce; ++p) {
                        const float x = (PF && a.append && p == start)
                                            ? x_first
                                            : load_in(src, a.dtype, in_base + (int64_t)(p - start) * D + c);
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
// Delta format.  LPC lanes per closed loop (1 or 2): the lanes of a loop own
// one 32-channel block of one tensor of one keyframe group of one (batch
// entry, kv head), lane u of them channels 32/LPC u .. 32/LPC (u + 1) - 1,
// and run the group's positions in order with their channels in registers.
// The block rule's signed element of largest magnitude is a scan in channel
// order with a strict comparison, which keeps the lowest index on ties, as
// the rule states: a pairwise tree inside the lane, then (LPC 2) the same
// comparison between the two halves, lower channels on the left.  Lane l of
// a warp takes part l % LPC of block (l / LPC) & 3 of tensor (l / 4 LPC) & 1
// of group (4 / LPC) q + l / 8 LPC, q the warp's group chunk.  The next
// position's inputs are loaded before the current position is quantised.
// Every quantiser step is one IEEE binary32 operation in the order of
// quant_lane.  Two lanes per loop serve caches with few loops per GPU (long
// keyframe groups, small batches).
// ---------------------------------------------------------------------------
constexpr int ENC_WARPS = 4;
// Closed loops (group x tensor x block) from which an append uses the
// one-lane-per-loop kernel: about two resident waves of its lanes on 148
// SMs.  Encodes always use this kernel, with two lanes per loop below one
// resident wave of loops.
constexpr int64_t kLaneKernelMinChains = 148 * 12 * 32 * 2;
constexpr int64_t kOneLanePerLoopMinChains = 148 * 12 * 32;

// CH consecutive inputs of one block at one position, as raw words (fp32: CH
// words; fp16 / bf16: CH / 2 words of two halves).
template <int DT, int CH>
struct EncRow {
    static constexpr int NW = DT == DKV_F32 ? CH : CH / 2;
    uint32_t w[NW];
    __device__ inline void load(const void *src, int64_t elem) {
        const uint4 *p = reinterpret_cast<const uint4 *>(
            static_cast<const uint8_t *>(src) + elem * (DT == DKV_F32 ? 4 : 2));
#pragma unroll
        for (int k = 0; k < NW / 4; ++k) {
            const uint4 v = __ldg(p + k);
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
        }
    }
    __device__ inline float get(int c) const {
        if (DT == DKV_F32) return __uint_as_float(w[c]);
        const uint32_t u = w[c >> 1];
        const unsigned short h = (c & 1) ? (unsigned short)(u >> 16) : (unsigned short)(u & 0xffffu);
        if (DT == DKV_F16) return __half2float(__ushort_as_half(h));
        return __bfloat162float(__ushort_as_bfloat16(h));
    }
};

template <int DT, int LPC>
__global__ void __launch_bounds__(ENC_WARPS * 32) encode_delta_kernel(EncodeArgs a, int NQ) {
    static_assert(LPC == 1 || LPC == 2, "one or two lanes per closed loop");
    constexpr int CH = 32 / LPC;              // channels per lane
    constexpr int GW = 4 / LPC;               // groups per warp
    const CacheView &cv = a.cv;
    const int lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * ENC_WARPS + (threadIdx.x >> 5);
    const int kf = cv.kf;
    if (item < (int64_t)cv.B * cv.Hkv * NQ) {
        const int qd = (int)(item % NQ);
        const int bh = (int)(item / NQ);
        const int b = bh / cv.Hkv, kvh = bh % cv.Hkv;
        const int u = lane % LPC, j = (lane / LPC) & 3, t = (lane / (4 * LPC)) & 1;
        const int gi = GW * qd + lane / (8 * LPC);
        // the lanes of one loop, for their exchanges (LPC 2)
        const unsigned pair = LPC == 2 ? 3u << (lane & ~1) : 1u << lane;
        int start, n;
        encode_range(a, b, start, n);
        const int parity = cv.header[2] & 1;
        const int64_t slot = (int64_t)cv.B * cv.Hkv * 2 * D;
        const int64_t sb = (((int64_t)b * cv.Hkv + kvh) * 2 + t) * D + 32 * j + CH * u;
        const float *st_old = cv.state + parity * slot + sb;
        float *st_new = cv.state + (parity ^ 1) * slot + sb;
        // checked build: the block's 32 state channels in both slots (the same
        // test in both lanes of a loop); outside, the loop is skipped (every
        // thread still reaches the grid's last-block step below)
        const bool st_in = !DKV_CHECKED ||
                           (state_ok(cv, st_old - CH * u, 32) && state_ok(cv, st_new - CH * u, 32));
        if (n < 0 && qd == 0 && kvh == 0 && lane == 0)
            set_status(cv.header, n == -2 ? DKV_DEV_CAPACITY : DKV_DEV_BAD_SEQLEN);
        if (!st_in) {
            // checked build: state outside its buffer, nothing read or written
        } else if (n <= 0) {
            if (gi == 0) {                         // nothing written: carry the state over
#pragma unroll
                for (int c = 0; c < CH; ++c) st_new[c] = a.append ? st_old[c] : 0.0f;
            }
        } else {
            const int g = start / kf + gi;
            const int p0 = max(start, g * kf), p1 = min(start + n, (g + 1) * kf);
            const bool last = p1 == start + n;
            uint8_t *rec = p0 < p1 ? rec_ptr(cv, b, kvh, g) : nullptr;
            if (rec && !rec_ok(cv, rec, cv.rec_bytes)) rec = nullptr;   // checked build
            bool in_ok = true;
            if (DKV_CHECKED && p0 < p1) {
                // the block's input rows [p0, p1) (the same test in both lanes)
                const int es = DT == DKV_F32 ? 4 : 2;
                const int64_t row = (((int64_t)b * cv.Hkv + kvh) * a.T_in - start + p0) * D + 32 * j;
                in_ok = range_ok(cv.header, static_cast<const uint8_t *>(t ? a.V : a.K) + row * es,
                                 ((int64_t)(p1 - p0 - 1) * D + 32) * es, t ? a.V : a.K,
                                 (int64_t)cv.B * cv.Hkv * a.T_in * D * es);
            }
            if (!in_ok) {
                // checked build: input outside its buffer, nothing written
            } else if (p0 < p1 && !rec) {
                // bad block-table entry (flagged by rec_ptr): nothing written
                if (last) {
#pragma unroll
                    for (int c = 0; c < CH; ++c) st_new[c] = (p0 % kf) ? st_old[c] : 0.0f;
                }
            } else if (p0 < p1) {
                const void *src = t ? a.V : a.K;
                const int64_t base =
                    (((int64_t)b * cv.Hkv + kvh) * a.T_in - start) * D + 32 * j + CH * u;
                float xh[CH];
#pragma unroll
                for (int c = 0; c < CH; ++c) xh[c] = (p0 % kf) ? st_old[c] : 0.0f;
                uint8_t *scl = rec + KF_BYTES + t * 8 + 2 * j;
                uint8_t *nib = rec + KF_BYTES + (int64_t)(kf - 1) * SC_BYTES +
                               (int64_t)t * (kf - 1) * NIB_BYTES;
                EncRow<DT, CH> cur, nxt;
                cur.load(src, base + (int64_t)p0 * D);
#pragma unroll 1
                for (int p = p0; p < p1; ++p) {
                    if (p + 1 < p1) nxt.load(src, base + (int64_t)(p + 1) * D);
                    const int di = p - g * kf;      // 0: keyframe; else delta di - 1
                    if (di == 0) {
                        // keyframe: fp16 values at their permuted halfword slots
                        __half h[CH];
#pragma unroll
                        for (int c = 0; c < CH; ++c) {
                            h[c] = __float2half_rn(cur.get(c));
                            xh[c] = __half2float(h[c]);
                        }
                        __half *kfr = reinterpret_cast<__half *>(rec + t * 256);
                        if (t == 0) {
                            // halfword t4 * 32 + 8 j + 4 s + 2 e + hh = channel 16 s + 8 e + 2 t4 + hh;
                            // lane u holds the channels with s = u (LPC 2)
#pragma unroll
                            for (int t4 = 0; t4 < 4; ++t4) {
                                uint32_t w4[4];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const int s2 = k >> 1, e = k & 1;
                                    const int c0 = 16 * (LPC == 1 ? s2 : 0) + 8 * e + 2 * t4;
                                    w4[k] = (uint32_t)__half_as_ushort(h[c0]) |
                                            ((uint32_t)__half_as_ushort(h[c0 + 1]) << 16);
                                }
                                if (LPC == 1)
                                    *reinterpret_cast<uint4 *>(kfr + t4 * 32 + 8 * j) =
                                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                                else   // halfwords 4 u + 0..3; w4[0..1] hold s = 0 of this lane's view
                                    *reinterpret_cast<uint2 *>(kfr + t4 * 32 + 8 * j + 4 * u) =
                                        make_uint2(w4[0], w4[1]);
                            }
                        } else {
                            // halfword gg * 16 + 4 j + 2 v + e = channel 16 v + gg + 8 e;
                            // lane u holds v = u (LPC 2)
#pragma unroll
                            for (int gg = 0; gg < 8; ++gg) {
                                const uint32_t w0 = (uint32_t)__half_as_ushort(h[gg]) |
                                                    ((uint32_t)__half_as_ushort(h[gg + 8]) << 16);
                                if (LPC == 1) {
                                    const uint32_t w1 = (uint32_t)__half_as_ushort(h[16 + gg]) |
                                                        ((uint32_t)__half_as_ushort(h[24 + gg]) << 16);
                                    *reinterpret_cast<uint2 *>(kfr + gg * 16 + 4 * j) =
                                        make_uint2(w0, w1);
                                } else {
                                    *reinterpret_cast<uint32_t *>(kfr + gg * 16 + 4 * j + 2 * u) = w0;
                                }
                            }
                        }
                    } else {
                        float dl[CH];
#pragma unroll
                        for (int c = 0; c < CH; ++c) dl[c] = __fsub_rn(cur.get(c), xh[c]);
                        // the signed element of largest magnitude, lowest index on
                        // ties: a pairwise tree that keeps the left (lower-index)
                        // element unless the right one is strictly larger
                        float ta[CH / 2], tm[CH / 2];
#pragma unroll
                        for (int i = 0; i < CH / 2; ++i) {
                            const float l = fabsf(dl[2 * i]), r = fabsf(dl[2 * i + 1]);
                            const bool right = r > l;
                            ta[i] = right ? r : l;
                            tm[i] = right ? dl[2 * i + 1] : dl[2 * i];
                        }
#pragma unroll
                        for (int w = CH / 4; w >= 1; w >>= 1)
#pragma unroll
                            for (int i = 0; i < w; ++i) {
                                const bool right = ta[2 * i + 1] > ta[2 * i];
                                tm[i] = right ? tm[2 * i + 1] : tm[2 * i];
                                ta[i] = right ? ta[2 * i + 1] : ta[2 * i];
                            }
                        float m = tm[0];
                        if (LPC == 2) {
                            // the two halves: the upper channels (lane u = 1)
                            // win only when strictly larger
                            const float ao = __shfl_xor_sync(pair, ta[0], 1);
                            const float mo = __shfl_xor_sync(pair, m, 1);
                            const float al = u ? ao : ta[0], ml = u ? mo : m;
                            const float ar = u ? ta[0] : ao, mr = u ? m : mo;
                            m = ar > al ? mr : ml;
                        }
                        const __half d16 = __float2half_rn(__fmul_rn(m, -0.125f));
                        const float d = __half2float(d16);
                        const bool z = d == 0.0f;
                        const float dd = z ? 1.0f : d;
                        const float rd = __frcp_rn(dd);      // one reciprocal per block and position
                        uint32_t code[CH];
#pragma unroll
                        for (int c = 0; c < CH; ++c) {
                            const int cc =
                                (int)truncf(__fadd_rn(div_rn_markstein(dl[c], dd, rd), 8.5f));
                            code[c] = z ? 8u : (uint32_t)min(15, max(0, cc));
                            xh[c] = __fadd_rn(xh[c], __fmul_rn((float)((int)code[c] - 8), d));
                        }
                        uint8_t *row = nib + (int64_t)(di - 1) * NIB_BYTES;
                        if (t == 0) {
                            // word t4 * 4 + j, nibble 4 hh + 2 s + e = channel 16 s + 8 e + 2 t4 + hh;
                            // lane u fills the nibbles with s = u (LPC 2)
#pragma unroll
                            for (int t4 = 0; t4 < 4; ++t4) {
                                uint32_t wd = 0;
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const int hh = i >> 2, s2 = (i >> 1) & 1, e = i & 1;
                                    if (LPC == 1)
                                        wd |= code[16 * s2 + 8 * e + 2 * t4 + hh] << (4 * i);
                                    else if (s2 == 0)
                                        wd |= code[8 * e + 2 * t4 + hh] << (4 * i + 8 * u);
                                }
                                if (LPC == 2) wd |= __shfl_xor_sync(pair, wd, 1);
                                if (u == 0) reinterpret_cast<uint32_t *>(row)[t4 * 4 + j] = wd;
                            }
                        } else {
                            // byte gg * 8 + 2 j + v = channel 16 v + gg (low) | 16 v + gg + 8 (high);
                            // lane u fills byte v = u (LPC 2)
#pragma unroll
                            for (int gg = 0; gg < 8; ++gg) {
                                uint32_t bb = code[gg] | (code[gg + 8] << 4);
                                if (LPC == 1) {
                                    bb |= (code[16 + gg] | (code[24 + gg] << 4)) << 8;
                                } else {
                                    bb <<= 8 * u;
                                    bb |= __shfl_xor_sync(pair, bb, 1);
                                }
                                if (u == 0)
                                    *reinterpret_cast<uint16_t *>(row + gg * 8 + 2 * j) = (uint16_t)bb;
                            }
                        }
                        if (u == 0) *reinterpret_cast<__half *>(scl + (int64_t)(di - 1) * SC_BYTES) = d16;
                    }
                    if (p + 1 < p1) cur = nxt;
                }
                if (last) {
#pragma unroll
                    for (int c = 0; c < CH; c += 4)
                        *reinterpret_cast<float4 *>(st_new + c) =
                            make_float4(xh[c], xh[c + 1], xh[c + 2], xh[c + 3]);
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
// Test support: the encoder's quotient against __fdiv_rn.  Block x = one fp16
// bit pattern of the divisor (every finite non-zero one); each thread takes
// multipliers u_i and checks a = RN(u_i b) and its two neighbours.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) division_check_kernel(const float *u, int n,
                                                             unsigned long long *bad) {
    const uint16_t hb = (uint16_t)blockIdx.x;
    const __half h = __ushort_as_half(hb);
    const float b = __half2float(h);
    if (!(b != 0.0f) || isinf(b) || isnan(b)) return;     // uniform over the block
    const float r = __frcp_rn(b);
    unsigned long long local = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float a0 = __fmul_rn(u[i], b);
        const float as[3] = {a0, nextafterf(a0, INFINITY), nextafterf(a0, -INFINITY)};
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const float x = __fdiv_rn(as[k], b), y = div_rn_markstein(as[k], b, r);
            // the bits where the quotient is normal; the code it gives always
            const bool normal = fabsf(x) >= 1.17549435e-38f;
            const int cx = min(15, max(0, (int)truncf(__fadd_rn(x, 8.5f))));
            const int cy = min(15, max(0, (int)truncf(__fadd_rn(y, 8.5f))));
            if ((normal && __float_as_uint(x) != __float_as_uint(y)) || cx != cy) ++local;
        }
    }
    if (local) atomicAdd(bad, local);
}

cudaError_t launch_division_check(const float *u, int n, unsigned long long *bad,
                                  cudaStream_t st) {
    division_check_kernel<<<65536, 256, 0, st>>>(u, n, bad);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_encode(const CacheView &cv, const void *K, const void *V, int dtype,
                          const int32_t *seq_lens, int T_in, int append, cudaStream_t st) {
    EncodeArgs a{cv, K, V, dtype, seq_lens, T_in, append};
    // groups a batch entry's range can touch (an append may start mid-group)
    const int NG = (T_in + cv.kf - 1) / cv.kf + (append ? 1 : 0);
    if (cv.fmt == DKV_FMT_DELTA &&
        (!append || (int64_t)cv.B * cv.Hkv * NG * 8 >= kLaneKernelMinChains)) {
        // an encode, or an append with enough closed loops to fill the GPU one
        // lane each; an encode with fewer than a resident wave of loops takes
        // two lanes per loop.  4 / LPC groups per warp.
        const int64_t chains = (int64_t)cv.B * cv.Hkv * NG * 8;
        const int lpc = (!append && chains < kOneLanePerLoopMinChains) ? 2 : 1;
        const int GW = 4 / lpc;
        const int NQ = (NG + GW - 1) / GW;
        const int64_t warps = (int64_t)cv.B * cv.Hkv * NQ;
        const int64_t ctas = (warps + ENC_WARPS - 1) / ENC_WARPS;
        if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
        const unsigned grid = (unsigned)ctas, blk = ENC_WARPS * 32;
        if (lpc == 2) {
            if (dtype == DKV_F32) encode_delta_kernel<DKV_F32, 2><<<grid, blk, 0, st>>>(a, NQ);
            else if (dtype == DKV_F16) encode_delta_kernel<DKV_F16, 2><<<grid, blk, 0, st>>>(a, NQ);
            else encode_delta_kernel<DKV_BF16, 2><<<grid, blk, 0, st>>>(a, NQ);
        } else {
            if (dtype == DKV_F32) encode_delta_kernel<DKV_F32, 1><<<grid, blk, 0, st>>>(a, NQ);
            else if (dtype == DKV_F16) encode_delta_kernel<DKV_F16, 1><<<grid, blk, 0, st>>>(a, NQ);
            else encode_delta_kernel<DKV_BF16, 1><<<grid, blk, 0, st>>>(a, NQ);
        }
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
        case DKV_FMT_DELTA: return launch_pdl(encode_kernel<DKV_FMT_DELTA>, grid, dim3(128), 0, st, a);
        case DKV_FMT_Q4_0: return launch_pdl(encode_kernel<DKV_FMT_Q4_0>, grid, dim3(128), 0, st, a);
        default: return launch_pdl(encode_kernel<DKV_FMT_FP16>, grid, dim3(128), 0, st, a);
    }
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
