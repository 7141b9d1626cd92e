// dkv_common.cuh -- shared device-side definitions of the Delta-KV library:
// the in-HBM layout of the three cache formats, the channel permutations that
// put each thread's tensor-core fragment in one contiguous chunk, and thin
// wrappers over the sm_100a PTX the kernels use (mbarrier, bulk async copy,
// mma.sync, prmt).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/dkv.h"

namespace dkv {

constexpr int D = 128;          // head_dim
constexpr int NB = 4;           // 32-channel quantisation blocks per token
constexpr int SEG = 32;         // positions per pipeline stage
constexpr int KF_BYTES = 512;   // K keyframe (256 B) followed by V keyframe (256 B)
constexpr int SC_BYTES = 16;    // per position: dK[4] then dV[4], fp16
constexpr int NIB_BYTES = 64;   // per position per tensor: 128 nibbles
constexpr int POS_Q4 = SC_BYTES + 2 * NIB_BYTES;   // 144 B per position
constexpr int POS_F16 = 2 * D * 2;                 // 512 B per position

// ---------------------------------------------------------------------------
// Layout of one sequence (one batch entry, one kv head):
//  DELTA: groups of kf positions, each a contiguous record
//           [K kf 256 B][V kf 256 B][scales (kf-1) x 16 B]
//           [K nibbles (kf-1) x 64 B][V nibbles (kf-1) x 64 B]
//         record g holds positions g*kf .. g*kf+kf-1; delta i of the record is
//         position g*kf + 1 + i.
//  Q4_0:  [scales cap x 16 B][K nibbles cap x 64 B][V nibbles cap x 64 B]
//  FP16:  [K cap x 256 B][V cap x 256 B]
// Every section size and offset is a multiple of 16 B, so 1-D bulk copies
// (which need 16-B aligned addresses and sizes) can move any run of them.
// ---------------------------------------------------------------------------
__host__ __device__ inline int64_t delta_rec_bytes(int kf) {
    return (int64_t)KF_BYTES + (int64_t)(kf - 1) * POS_Q4;
}

// ---------------------------------------------------------------------------
// Channel permutations.  With g = lane / 4 and t = lane % 4:
//  K nibbles of one position: 16 words; word (t*4 + j) holds block j's
//   channels {32j + 16s + 8e + 2t + h}, nibble index i = 4h + 2s + e.  A
//   mask with 0x000F000F of the word (or of the word >> 8 for s = 1) yields the
//   fp16x2 pair of channels (2t, 2t+1) of k-step 2j+s; 0x00F000F0 yields
//   (2t+8, 2t+9): exactly the B fragment of mma.m16n8k16 for column g.
//  V nibbles of one position: 8 chunks of 8 B; byte (g*8 + mt) holds channel
//   16mt + g (low nibble) and 16mt + g + 8 (high nibble): the rows thread g
//   owns in the A fragment of m-tile mt.
//  K keyframe / FP16 K values: halfword (t*32 + 4kk + 2e + h) = channel
//   16kk + 8e + 2t + h (the B fragment pairs of column g = 0).
//  V keyframe / FP16 V values: halfword (g*16 + 2mt + e) = channel
//   16mt + g + 8e.
// ---------------------------------------------------------------------------
__host__ __device__ inline void k_nib_pos(int c, int &byte, int &shift) {
    int j = c >> 5, r = c & 31, s = r >> 4, r2 = r & 15, e = r2 >> 3, r3 = r2 & 7;
    int t = r3 >> 1, h = r3 & 1;
    int word = t * 4 + j, i = 4 * h + 2 * s + e;
    byte = word * 4 + (i >> 1);
    shift = 4 * (i & 1);
}
__host__ __device__ inline void v_nib_pos(int c, int &byte, int &shift) {
    int mt = c >> 4, r = c & 15, g = r & 7, hi = r >> 3;
    byte = g * 8 + mt;
    shift = 4 * hi;
}
__host__ __device__ inline int k_half_idx(int c) {
    int kk = c >> 4, r = c & 15, e = r >> 3, t = (r & 7) >> 1, h = r & 1;
    return t * 32 + 4 * kk + 2 * e + h;
}
__host__ __device__ inline int v_half_idx(int c) {
    int mt = c >> 4, r = c & 15, g = r & 7, e = r >> 3;
    return g * 16 + 2 * mt + e;
}

// Channel held by nibble i (0..7) of word w (0..15) of one position's nibble
// row of tensor t: the inverse of k_nib_pos (K) / v_nib_pos (V).
__host__ __device__ inline int nib_channel(int t, int w, int i) {
    if (t == 0) {
        const int tt = w >> 2, j = w & 3, h = i >> 2, s2 = (i >> 1) & 1, e = i & 1;
        return 32 * j + 16 * s2 + 8 * e + 2 * tt + h;
    }
    const int g = w >> 1, u = w & 1, mt = 4 * u + (i >> 1);
    return 16 * mt + g + 8 * (i & 1);
}

// Device-side cache view passed by value to kernels.
struct CacheView {
    uint8_t *data;
    int64_t data_bytes;    // bytes of the data area (contiguous caches)
    float *state;          // [2][B][Hkv][2][D]
    int32_t *seqlen;       // [B]
    int32_t *header;       // {status, counter, parity, reserved}
    int64_t seq_stride;
    int64_t rec_bytes;
    int32_t B, Hkv, kf, cap, fmt, n_groups;
    // paged (delta format): pg = groups per page (0: contiguous)
    uint8_t *pool;
    const int32_t *bt;     // [B][maxp] page indices
    int64_t page_bytes, n_pages;
    int32_t pg, maxp;
    // fused append + decode: tokens each sequence takes in this call (0:
    // none); a sequence whose tokens fit is decoded at its stored length + this
    int32_t len_add;
};

__device__ inline void set_status(int32_t *header, int bits) {
    atomicOr(reinterpret_cast<int *>(header), bits);
}

// Checked builds (DKV_CHECKED=1, for tests): every computed global memory
// range is tested against the buffer it must lie in; a range outside sets
// DKV_DEV_BOUNDS and the access is skipped.  In normal builds the tests are
// compiled out.
#ifndef DKV_CHECKED
#define DKV_CHECKED 0
#endif
__device__ inline bool range_ok(int32_t *header, const void *p, int64_t n, const void *lo,
                                int64_t size) {
    if constexpr (DKV_CHECKED == 0) {
        return true;
    } else {
        const uint8_t *a = static_cast<const uint8_t *>(p), *b = static_cast<const uint8_t *>(lo);
        const bool ok = n >= 0 && a >= b && a + n <= b + size;
        if (!ok) set_status(header, DKV_DEV_BOUNDS);
        return ok;
    }
}
// n bytes at p inside the cache's records: the data area, or the page pool
__device__ inline bool rec_ok(const CacheView &cv, const void *p, int64_t n) {
    if constexpr (DKV_CHECKED == 0) return true;
    return cv.pg ? range_ok(cv.header, p, n, cv.pool, cv.n_pages * cv.page_bytes)
                 : range_ok(cv.header, p, n, cv.data, cv.data_bytes);
}
// n floats at p inside the reconstruction state (both slots)
__device__ inline bool state_ok(const CacheView &cv, const float *p, int64_t n) {
    if constexpr (DKV_CHECKED == 0) return true;
    return range_ok(cv.header, p, n * 4, cv.state, (int64_t)2 * cv.B * cv.Hkv * 2 * D * 4);
}

// Record g (delta format) of sequence (b, kvh): contiguous, or through the
// block table (PAGED); nullptr (and DKV_DEV_BAD_PAGE) for an entry outside the
// pool.
template <bool PAGED>
__device__ inline uint8_t *rec_ptr(const CacheView &cv, int b, int kvh, int g) {
    if (!PAGED)
        return cv.data + ((int64_t)b * cv.Hkv + kvh) * cv.seq_stride + (int64_t)g * cv.rec_bytes;
    const int page = cv.bt[(int64_t)b * cv.maxp + g / cv.pg];
    if (page < 0 || page >= cv.n_pages) {
        set_status(cv.header, DKV_DEV_BAD_PAGE);
        return nullptr;
    }
    return cv.pool + (int64_t)page * cv.page_bytes + ((int64_t)kvh * cv.pg + g % cv.pg) * cv.rec_bytes;
}
__device__ inline uint8_t *rec_ptr(const CacheView &cv, int b, int kvh, int g) {
    return cv.pg ? rec_ptr<true>(cv, b, kvh, g) : rec_ptr<false>(cv, b, kvh, g);
}

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ inline uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline void mbar_init(uint64_t *bar, int count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ inline void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ inline void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// orders this thread's generic-proxy global stores before later bulk copies
__device__ inline void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;\n" ::: "memory");
}

// Programmatic dependent launch.  The library's step kernels (append, decode
// split, merge) are launched with programmatic stream serialization, so each
// may be scheduled while the kernel before it in the stream still runs.
// pdl_wait() returns once every kernel before it in the stream has completed
// and its global writes are visible: each of those kernels calls it before its
// first global access, so the order of the stream holds for memory.  It
// returns at once in a launch without that attribute.  pdl_trigger() lets the
// next such kernel be scheduled; it orders nothing.
__device__ inline void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ inline void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// host side: a launch with programmatic stream serialization allowed
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}
__device__ inline void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ inline bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after ~2^31 cycles (about a second) and returns false.
__device__ inline bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > (1ll << 31)) return false;
    }
}
// 1-D bulk async copy global -> shared, completion counted on `bar`.
__device__ inline void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ inline uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ inline uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    return (a & mask) | orv;  // compiles to one LOP3
}
__device__ inline uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ inline __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

__device__ inline uint32_t pack_h2(float lo, float hi) {
    return h2_as_u32(__floats2half2_rn(lo, hi));
}
__device__ inline float h_lo(uint32_t u) { return __low2float(u32_as_h2(u)); }
__device__ inline float h_hi(uint32_t u) { return __high2float(u32_as_h2(u)); }
// 8x8 transpose of b16 elements across the warp (thread t holds row t / 4,
// columns 2 (t % 4) and 2 (t % 4) + 1).
__device__ inline uint32_t movm_t(uint32_t a) {
    uint32_t d;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
    return d;
}

// D = A(16x16 f16, row) * B(16x8 f16, col) + C, fp32 accumulate.
__device__ inline void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ldmatrix: four 8x8 b16 tiles from shared memory (lane l gives the address
// of row l % 8 of tile l / 8); .trans delivers each tile transposed.
__device__ inline void ldsm_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ inline void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

// The fp16 bit pattern of 1024.0 in both halves, as a register value the
// compiler cannot fold: OR-ing a nibble into it needs the mask as the one
// immediate operand of a single LOP3 and this value in a register.
__device__ inline uint32_t magic_1024x2() {
    uint32_t r;
    asm volatile("mov.b32 %0, 0x64006400;\n" : "=r"(r));
    return r;
}
// fp16 64.0 in both halves: its ulp is 1/16, so a nibble OR-ed into mantissa
// bits 4-7 reads as 64 + n exactly.
__device__ inline uint32_t magic_64x2() {
    uint32_t r;
    asm volatile("mov.b32 %0, 0x54005400;\n" : "=r"(r));
    return r;
}

// Biased dequantisation: one LOP3 per fp16x2 pair.  The pairs read 1024 + n
// (nibbles at bits 0-3 / 16-19, over the 1024 magic) and 64 + n (bits 4-7 /
// 20-23, over the 64 magic); dq_word / dq_pair subtract 1032 and 72.
__device__ inline void dq_word_biased(uint32_t w, uint32_t m1024, uint32_t m64, uint32_t &p0,
                                      uint32_t &p1, uint32_t &p2, uint32_t &p3);
__device__ inline void dq_pair_biased(uint32_t w, uint32_t m1024, uint32_t m64, uint32_t &lo,
                                      uint32_t &hi);
// (a & MASK) | c in one LOP3 (LUT 0xEA).
template <uint32_t MASK>
__device__ inline uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(d) : "r"(a), "n"(MASK), "r"(c));
    return d;
}
// fp16x2 helpers on raw 32-bit registers
__device__ inline uint32_t hsub2_1032(uint32_t a) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(0x64086408u));
    return d;
}
__device__ inline uint32_t hsub2_72(uint32_t a) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(0x54805480u));
    return d;
}

__device__ inline void dq_word_biased(uint32_t w, uint32_t m1024, uint32_t m64, uint32_t &p0,
                                      uint32_t &p1, uint32_t &p2, uint32_t &p3) {
    const uint32_t w8 = w >> 8;
    p0 = and_or<0x000F000Fu>(w, m1024);
    p1 = and_or<0x00F000F0u>(w, m64);
    p2 = and_or<0x000F000Fu>(w8, m1024);
    p3 = and_or<0x00F000F0u>(w8, m64);
}
__device__ inline void dq_pair_biased(uint32_t w, uint32_t m1024, uint32_t m64, uint32_t &lo,
                                      uint32_t &hi) {
    lo = and_or<0x000F000Fu>(w, m1024);
    hi = and_or<0x00F000F0u>(w, m64);
}

// Exact dequantisation of the 4 nibble pairs of one 32-bit word (pairs (bits
// 0-3,16-19), (4-7,20-23), (8-11,24-27), (12-15,28-31)) to fp16x2 values
// code - 8: (1024 + n) - 1032 for the low nibbles, (64 + n) - 72 for the high.
__device__ inline void dq_word(uint32_t w, uint32_t m1024, uint32_t m64, uint32_t &p0,
                               uint32_t &p1, uint32_t &p2, uint32_t &p3) {
    dq_word_biased(w, m1024, m64, p0, p1, p2, p3);
    p0 = hsub2_1032(p0);
    p1 = hsub2_72(p1);
    p2 = hsub2_1032(p2);
    p3 = hsub2_72(p3);
}

// The low-nibble pair (bits 0-3, 16-19) and the high-nibble pair (bits 4-7,
// 20-23) of one 32-bit word as exact fp16x2 values code - 8.
__device__ inline void dq_pair(uint32_t w, uint32_t m1024, uint32_t m64, uint32_t &lo,
                               uint32_t &hi) {
    dq_pair_biased(w, m1024, m64, lo, hi);
    lo = hsub2_1032(lo);
    hi = hsub2_72(hi);
}

// ---------------------------------------------------------------------------
// The quantiser, shared by the encoder and the fused append of the decode
// ---------------------------------------------------------------------------
__device__ inline float load_in(const void *p, int dtype, int64_t i) {
    if (dtype == DKV_F32) return static_cast<const float *>(p)[i];
    if (dtype == DKV_F16) return __half2float(static_cast<const __half *>(p)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

// The Q4_0 block rule for the 32 lanes of one warp (lane = element).
// Returns the code; *d16 receives the block scale (same value in every lane).
__device__ inline int quant_lane(float v, __half *d16_out) {
    uint32_t a = __float_as_uint(v) & 0x7fffffffu;
    uint32_t mx = __reduce_max_sync(0xffffffffu, a);
    uint32_t ball = __ballot_sync(0xffffffffu, a == mx);
    float m = __shfl_sync(0xffffffffu, v, __ffs(ball) - 1);  // lowest index on ties
    float d32 = __fmul_rn(m, -0.125f);   // = m / -8 exactly: one rounding of the same real value
    __half d16 = __float2half_rn(d32);
    float d = __half2float(d16);
    *d16_out = d16;
    if (d == 0.0f) return 8;
    float q = __fdiv_rn(v, d);
    float u = __fadd_rn(q, 8.5f);
    int c = (int)truncf(u);
    return min(15, max(0, c));
}

// Correctly rounded binary32 quotient a / b, given r = RN(1/b) (one
// correctly rounded reciprocal serves every quotient by the same b).  One
// refinement q1 = q0 + r (a - b q0) makes q1 faithful (relative error about
// 4u^2 before rounding, u = 2^-24); then, with q1 faithful, the residual
// a - b q1 is exact in one fused multiply-add and RN(q1 + r (a - b q1)) is
// RN(a / b): the correction theorem of P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990.  Holds without overflow or underflow; a quotient below
// the normal range (only for a subnormal dividend here) may differ in its last
// bit, and feeds code 8 either way.  Checked against __fdiv_rn over every fp16
// divisor by dkv_debug_division_check.
__device__ inline float div_rn_markstein(float a, float b, float r) {
    const float q0 = __fmul_rn(a, r);
    const float q1 = __fmaf_rn(__fmaf_rn(-b, q0, a), r, q0);
    return __fmaf_rn(__fmaf_rn(-b, q1, a), r, q1);
}

// The block rule on NC independent blocks at once (element lane of each),
// written phase by phase -- every block's reduction, then every block's
// vote, ... -- so the warp-wide steps of the blocks overlap instead of
// running one block after another.  Each block takes exactly the steps of
// quant_lane, in the same order.  A zero scale divides by 1 (the code is
// then 8 regardless), so no division ever sees a zero divisor.
template <int NC>
__device__ inline void quant_lanes(const float (&v)[NC], int (&code)[NC], __half (&d16)[NC]) {
    uint32_t a[NC], mx[NC], ball[NC];
    float m[NC], d[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) a[i] = __float_as_uint(v[i]) & 0x7fffffffu;
#pragma unroll
    for (int i = 0; i < NC; ++i) mx[i] = __reduce_max_sync(0xffffffffu, a[i]);
#pragma unroll
    for (int i = 0; i < NC; ++i) ball[i] = __ballot_sync(0xffffffffu, a[i] == mx[i]);
#pragma unroll
    for (int i = 0; i < NC; ++i) m[i] = __shfl_sync(0xffffffffu, v[i], __ffs(ball[i]) - 1);
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        d16[i] = __float2half_rn(__fmul_rn(m[i], -0.125f));
        d[i] = __half2float(d16[i]);
    }
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const bool z = d[i] == 0.0f;
        const float q = __fdiv_rn(v[i], z ? 1.0f : d[i]);
        const int c = (int)truncf(__fadd_rn(q, 8.5f));
        code[i] = z ? 8 : min(15, max(0, c));
    }
}

}  // namespace dkv
