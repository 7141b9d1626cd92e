// decode.cu -- one decode step of GQA attention over a Delta-KV cache (and
// over the fp16 / Q4_0 comparator caches), for sm_100a.
//
// The step (page "KV 캐시 벡터 양자화와 주의 보존 변환", section "KV 캐시가 왜
// 병목인가"): read every cached K/V from HBM, form q.k, softmax, A.V.  The read
// is the bottleneck, so the kernel streams the compressed cache exactly once
// and never materialises a reconstructed K or V.
//
// Reconstruction by linearity.  Inside a keyframe group with keyframe f
// (page "...Delta-KV", section "핵심 아이디어"),
//     k^_p = k_f + sum_{f<s<=p} delta^_s,  delta^_s = (code_s - 8) * d_s,
// so for every query head h
//     q_h . k^_p = sum_{s<=p} q_h . delta^_s      (position f carries q_h . k_f)
// is a prefix sum over positions of per-position dot products, and
//     sum_p w_hp v^_p = sum_s delta^_s * S_hs,     S_hs = sum_{p>=s} w_hp
// (position f carries v_f with S_hf = the group's total weight) is a sum of
// dequantised delta rows weighted by suffix sums of the softmax weights.  Both
// per-position products are dense tiles for the tensor cores:
//   K side  D[h][p] = sum_c q[h][c] * code[p][c]  per 32-channel block, m16n8k16
//           with heads as M (8 of 16 rows used) and positions as N;
//   V side  O[c][h] += sum_p code[p][c] * (S[h][p] * d[p][blk(c)]), m16n8k16
//           with channels as M, positions as K and heads as N.
// The K-side accumulator layout of a thread (head g, positions 2t, 2t+1) is
// exactly the V-side B-fragment layout, so the softmax weights flow from one
// MMA to the other without shuffles.
//
// Groups longer than one 32-position stage (kf > 32) use the equivalent
// forward form  sum_p w_p v^_p = W_g (v_f + R_g) - sum_s delta^_s E_s  with
// E_s the exclusive prefix of the weights inside the group and R_g the sum of
// the group's dequantised deltas (an extra MMA against the scales alone).
//
// Work split: the (sequence, group) units of all sequences are flattened and
// cut into equal contiguous ranges, one per warp of a persistent grid.  Each
// warp streams its range through its own ring of shared-memory stages filled
// by 1-D bulk async copies (cp.async.bulk + mbarrier), keeps an online-softmax
// state per sequence it touches, and writes one partial (max, sum, output)
// record per such sequence.  The merge kernel combines the partial records
// with a log-sum-exp.
#include <cstdint>

#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace dkv {

enum Mode { SUFFIX = 0, PREFIX = 1, PLAIN = 2 };

constexpr int WARPS = 4;                     // warps per CTA (independent pipelines)
constexpr int MAX_B = 1024;

template <int FMT> struct FmtCfg;
template <> struct FmtCfg<DKV_FMT_DELTA> { static constexpr int STAGE = 5120, NS = 3; };
template <> struct FmtCfg<DKV_FMT_Q4_0>  { static constexpr int STAGE = 5120, NS = 3; };
template <> struct FmtCfg<DKV_FMT_FP16>  { static constexpr int STAGE = 16384, NS = 2; };

// Stage layout (DELTA / Q4_0): [K kf 256][V kf 256][scales 32x16][K nib 32x64][V nib 32x64]
constexpr int ST_KF = 0, ST_SC = 512, ST_KN = 1024, ST_VN = 3072;

struct SplitArgs {
    CacheView cv;
    const void *Q;
    int q_dtype;
    int Hq, G, NHG;            // query heads, heads per kv head, head groups of 8
    float scale_log2;          // softmax_scale * log2(e)
    float *ws;                 // partial records
};

__host__ __device__ inline int units_of(int fmt, int kf, int len) {
    if (len <= 0) return 0;
    return fmt == DKV_FMT_DELTA ? (len + kf - 1) / kf : (len + SEG - 1) / SEG;
}

// Warp w of NW owns units [w*T/NW, (w+1)*T/NW).
__host__ __device__ inline int64_t range_start(int64_t w, int64_t NW, int64_t T) {
    return (w * T) / NW;
}
__host__ __device__ inline int64_t warp_of(int64_t x, int64_t NW, int64_t T) {
    return ((x + 1) * NW - 1) / T;
}

// Iterates the (unit, segment) stage items of one warp's range in order.
struct Cursor {
    int64_t x, x_end;          // flattened unit index, end of range
    int b, vs, g;              // batch entry, sequence within the batch entry, unit
    int units_b;               // units per sequence of batch entry b
    int len_b;                 // tokens of batch entry b
    int seg, nseg;             // segment within the unit
    __device__ bool valid() const { return x < x_end; }
};

__device__ inline int clamp_len(const CacheView &cv, int b) {
    int l = cv.seqlen[b];
    return (l < 0 || l > cv.cap) ? 0 : l;
}

__device__ inline int nseg_of(const CacheView &cv, int len, int g) {
    if (cv.fmt != DKV_FMT_DELTA) return 1;
    int glen = min(cv.kf, len - g * cv.kf);
    return (glen + SEG - 1) / SEG;
}

__device__ inline void cursor_seek(Cursor &c, const CacheView &cv, const int64_t *plan, int nvs) {
    // find b with plan[b] <= x < plan[b+1]
    int lo = 0, hi = cv.B;  // invariant plan[lo] <= x < plan[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (plan[mid] <= c.x) lo = mid; else hi = mid;
    }
    c.b = lo;
    c.len_b = clamp_len(cv, lo);
    c.units_b = units_of(cv.fmt, cv.kf, c.len_b);
    int64_t r = c.x - plan[lo];
    c.vs = (int)(r / c.units_b);
    c.g = (int)(r % c.units_b);
    c.seg = 0;
    c.nseg = nseg_of(cv, c.len_b, c.g);
    (void)nvs;
}

__device__ inline void cursor_next(Cursor &c, const CacheView &cv, int nvs) {
    if (++c.seg < c.nseg) return;
    c.seg = 0;
    ++c.x;
    if (!c.valid()) return;
    if (++c.g == c.units_b) {
        c.g = 0;
        if (++c.vs == nvs) {
            c.vs = 0;
            do {
                ++c.b;
                c.len_b = clamp_len(cv, c.b);
                c.units_b = units_of(cv.fmt, cv.kf, c.len_b);
            } while (c.units_b == 0);
        }
    }
    c.nseg = nseg_of(cv, c.len_b, c.g);
}

// Issue the bulk copies of one stage item (one lane).
template <int FMT>
__device__ inline void issue_stage(const CacheView &cv, const Cursor &c, int nvs_per_kv,
                                   uint8_t *stage, uint64_t *bar) {
    const int kvh = c.vs / nvs_per_kv;
    const uint8_t *sb = cv.data + ((int64_t)c.b * cv.Hkv + kvh) * cv.seq_stride;
    if (FMT == DKV_FMT_DELTA) {
        const int kf = cv.kf;
        const int glen = min(kf, c.len_b - c.g * kf);
        const int a = c.seg * SEG;
        const int npos = min(SEG, glen - a);
        const uint8_t *rec = sb + (int64_t)c.g * cv.rec_bytes;
        const uint8_t *scs = rec + KF_BYTES;
        const uint8_t *kns = scs + (int64_t)(kf - 1) * SC_BYTES;
        const uint8_t *vns = kns + (int64_t)(kf - 1) * NIB_BYTES;
        // slot s of the stage holds position a + s, i.e. delta index a + s - 1
        const int s0 = (a == 0) ? 1 : 0;       // slot 0 of segment 0 is the keyframe
        const int nd = npos - s0;
        const int di0 = a + s0 - 1;
        uint32_t bytes = (a == 0 ? KF_BYTES : 0) + nd * (SC_BYTES + 2 * NIB_BYTES);
        mbar_arrive_expect_tx(bar, bytes);
        if (a == 0) bulk_g2s(stage + ST_KF, rec, KF_BYTES, bar);
        if (nd > 0) {
            bulk_g2s(stage + ST_SC + s0 * SC_BYTES, scs + (int64_t)di0 * SC_BYTES, nd * SC_BYTES, bar);
            bulk_g2s(stage + ST_KN + s0 * NIB_BYTES, kns + (int64_t)di0 * NIB_BYTES,
                     nd * NIB_BYTES, bar);
            bulk_g2s(stage + ST_VN + s0 * NIB_BYTES, vns + (int64_t)di0 * NIB_BYTES,
                     nd * NIB_BYTES, bar);
        }
    } else if (FMT == DKV_FMT_Q4_0) {
        const int p0 = c.g * SEG;
        const int npos = min(SEG, c.len_b - p0);
        mbar_arrive_expect_tx(bar, npos * (SC_BYTES + 2 * NIB_BYTES));
        bulk_g2s(stage + ST_SC, sb + (int64_t)p0 * SC_BYTES, npos * SC_BYTES, bar);
        bulk_g2s(stage + ST_KN, sb + (int64_t)cv.cap * SC_BYTES + (int64_t)p0 * NIB_BYTES,
                 npos * NIB_BYTES, bar);
        bulk_g2s(stage + ST_VN, sb + (int64_t)cv.cap * (SC_BYTES + NIB_BYTES) + (int64_t)p0 * NIB_BYTES,
                 npos * NIB_BYTES, bar);
    } else {
        const int p0 = c.g * SEG;
        const int npos = min(SEG, c.len_b - p0);
        mbar_arrive_expect_tx(bar, npos * 512);
        bulk_g2s(stage, sb + (int64_t)p0 * 256, npos * 256, bar);
        bulk_g2s(stage + 8192, sb + (int64_t)cv.cap * 256 + (int64_t)p0 * 256, npos * 256, bar);
    }
}

__device__ inline uint32_t pack_h2(float lo, float hi) {
    return h2_as_u32(__floats2half2_rn(lo, hi));
}
__device__ inline float h_lo(uint32_t u) { return __low2float(u32_as_h2(u)); }
__device__ inline float h_hi(uint32_t u) { return __high2float(u32_as_h2(u)); }
__device__ inline uint32_t lds32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }
__device__ inline uint2 lds64(const uint8_t *p) { return *reinterpret_cast<const uint2 *>(p); }
__device__ inline uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }

__device__ inline float q_elem(const void *Q, int dt, int64_t i) {
    if (dt == DKV_F32) return static_cast<const float *>(Q)[i];
    if (dt == DKV_F16) return __half2float(static_cast<const __half *>(Q)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(Q)[i]);
}

// Inclusive scan over the 32 positions (8*nt + 2*t + e) of one head, held as
// x[nt][e] across the 4 lanes of a quad.  Returns the total (all lanes).
__device__ inline float quad_scan32(float (&x)[4][2], int t) {
    float tot[4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        x[nt][1] += x[nt][0];
        float own = x[nt][1];
        float inc = own;
        float u = __shfl_up_sync(0xffffffffu, inc, 1, 4);
        if (t >= 1) inc += u;
        u = __shfl_up_sync(0xffffffffu, inc, 2, 4);
        if (t >= 2) inc += u;
        float ex = inc - own;
        x[nt][0] += ex;
        x[nt][1] += ex;
        tot[nt] = __shfl_sync(0xffffffffu, inc, 3, 4);
    }
    float c1 = tot[0], c2 = c1 + tot[1], c3 = c2 + tot[2];
    x[1][0] += c1; x[1][1] += c1;
    x[2][0] += c2; x[2][1] += c2;
    x[3][0] += c3; x[3][1] += c3;
    return c3 + tot[3];
}

template <int FMT, int MODE>
__global__ void __launch_bounds__(WARPS * 32) split_kernel(SplitArgs A) {
    using Cfg = FmtCfg<FMT>;
    constexpr int NS = Cfg::NS, STAGE = Cfg::STAGE;
    extern __shared__ __align__(128) uint8_t smem[];
    int64_t *plan = reinterpret_cast<int64_t *>(smem);                       // [MAX_B + 1]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 8 * (MAX_B + 1));   // [WARPS][NS]
    uint8_t *stages = smem + 8 * (MAX_B + 1) + 8 * WARPS * NS + 64;          // 128-aligned below
    stages = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(stages) + 127) & ~uintptr_t(127));

    const CacheView &cv = A.cv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;          // quad row / column of the fragments
    const int nvs_per_kv = A.NHG;
    const int nvs = cv.Hkv * A.NHG;                    // sequences per batch entry

    // ---- plan: prefix over batch entries of units ------------------------
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int b = 0; b < cv.B; ++b) {
            plan[b] = acc;
            int l = cv.seqlen[b];
            if (l < 0 || l > cv.cap) {
                if (blockIdx.x == 0) set_status(cv.header, DKV_DEV_BAD_SEQLEN);
                l = 0;
            }
            acc += (int64_t)nvs * units_of(cv.fmt, cv.kf, l);
        }
        plan[cv.B] = acc;
    }
    uint64_t *mybar = bars + warp * NS;
    uint8_t *mystages = stages + (size_t)warp * NS * STAGE;
    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(mybar + s, 1);
        fence_mbar_init();
    }
    // zero the stages once so slots no copy has filled hold finite values
    for (int i = lane; i < NS * STAGE / 16; i += 32)
        reinterpret_cast<uint4 *>(mystages)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    __syncthreads();

    const int64_t total = plan[cv.B];
    const int64_t NW = (int64_t)gridDim.x * WARPS;
    const int64_t gw = (int64_t)blockIdx.x * WARPS + warp;
    if (total == 0) return;
    const int64_t r0 = range_start(gw, NW, total), r1 = range_start(gw + 1, NW, total);
    if (r0 >= r1) return;

    Cursor ic, cc;
    ic.x = r0; ic.x_end = r1;
    cursor_seek(ic, cv, plan, nvs);
    cc = ic;

    // prologue: fill the ring
    uint32_t phase = 0;                 // bit s = parity to wait for on stage s
#pragma unroll 1
    for (int s = 0; s < NS; ++s) {
        if (ic.valid()) {
            if (lane == 0) issue_stage<FMT>(cv, ic, nvs_per_kv, mystages + s * STAGE, mybar + s);
            cursor_next(ic, cv, nvs);
        }
    }

    bool dead = false;
    int stage_i = 0;

    // per-sequence state
    int cur_b = -1, cur_vs = -1;
    uint32_t qa[8][2];                  // A fragments of q (rows = heads)
    bool head_ok = false;
    float m_run = -1e30f, l_run = 0.f;
    float o[8][4];
    float racc[8][4];                   // PREFIX: sum of dequantised deltas of the group
    float dot_carry = 0.f, e_carry = 0.f;
    uint32_t vkf_keep[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { o[i][j] = 0.f; racc[i][j] = 0.f; }
#pragma unroll
    for (int i = 0; i < 8; ++i) vkf_keep[i] = 0;

    auto flush = [&]() {
        // write the partial record of the current sequence
        float l = l_run;
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int64_t vseq = ((int64_t)cur_b * cv.Hkv) * A.NHG + cur_vs;
        float *rec = A.ws + (gw + vseq) * PARTIAL_FLOATS;
        if (tq == 0) {
            rec[gq] = m_run;
            rec[8 + gq] = l;
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int c0 = 16 * mt + gq;
            rec[16 + (2 * tq) * 128 + c0] = o[mt][0];
            rec[16 + (2 * tq + 1) * 128 + c0] = o[mt][1];
            rec[16 + (2 * tq) * 128 + c0 + 8] = o[mt][2];
            rec[16 + (2 * tq + 1) * 128 + c0 + 8] = o[mt][3];
        }
    };

#pragma unroll 1
    while (cc.valid()) {
        // ---- sequence change: flush, load q --------------------------------
        if (cc.b != cur_b || cc.vs != cur_vs) {
            if (cur_b >= 0) flush();
            cur_b = cc.b; cur_vs = cc.vs;
            const int kvh = cc.vs / A.NHG, hg = cc.vs % A.NHG;
            const int hl = hg * 8 + gq;                  // head within the kv group
            head_ok = hl < A.G;
            const int64_t qrow = ((int64_t)cc.b * A.Hq + (int64_t)kvh * A.G + (head_ok ? hl : 0)) * D;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c = 16 * kk + 2 * tq;
                float q0 = 0.f, q1 = 0.f, q8 = 0.f, q9 = 0.f;
                if (head_ok) {
                    q0 = q_elem(A.Q, A.q_dtype, qrow + c);
                    q1 = q_elem(A.Q, A.q_dtype, qrow + c + 1);
                    q8 = q_elem(A.Q, A.q_dtype, qrow + c + 8);
                    q9 = q_elem(A.Q, A.q_dtype, qrow + c + 9);
                }
                qa[kk][0] = pack_h2(q0, q1);
                qa[kk][1] = pack_h2(q8, q9);
            }
            m_run = -1e30f; l_run = 0.f; dot_carry = 0.f; e_carry = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) { o[i][j] = 0.f; racc[i][j] = 0.f; }
        }

        // ---- wait for the stage -------------------------------------------
        uint8_t *st = mystages + stage_i * STAGE;
        if (!dead) {
            if (!mbar_wait_bounded(mybar + stage_i, (phase >> stage_i) & 1)) {
                dead = true;
                if (lane == 0) set_status(cv.header, DKV_DEV_TIMEOUT);
            }
        }
        dead = __any_sync(0xffffffffu, dead);
        phase ^= 1u << stage_i;

        if (!dead) {
            // positions of this stage: a + slot, slot < npos valid
            int a, npos;
            if (FMT == DKV_FMT_DELTA) {
                const int glen = min(cv.kf, cc.len_b - cc.g * cv.kf);
                a = cc.seg * SEG;
                npos = min(SEG, glen - a);
            } else {
                a = 0;
                npos = min(SEG, cc.len_b - cc.g * SEG);
            }
            const bool first_seg = (FMT == DKV_FMT_DELTA) && cc.seg == 0;
            const bool last_seg = cc.seg == cc.nseg - 1;

            // ================= K side: per-position dot products ============
            float x[4][2];
            uint32_t dvh[4][2][2];   // dV pairs (blocks 0|1, 2|3) per (nt, e)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int pc = 8 * nt + gq;            // position of this thread's B column
                uint32_t bf[8][2];
                if (FMT == DKV_FMT_FP16) {
                    const uint8_t *kp = st + pc * 256 + 64 * tq;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 v = lds128(kp + 16 * q4);
                        bf[2 * q4][0] = v.x; bf[2 * q4][1] = v.y;
                        bf[2 * q4 + 1][0] = v.z; bf[2 * q4 + 1][1] = v.w;
                    }
                } else {
                    uint4 kw = lds128(st + ST_KN + pc * NIB_BYTES + 16 * tq);
                    uint32_t ws4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dq_word(ws4[j], bf[2 * j][0], bf[2 * j][1], bf[2 * j + 1][0], bf[2 * j + 1][1]);
                    if (first_seg && nt == 0 && gq == 0) {
                        // position 0 is the keyframe: its fp16 values are the B column
                        const uint8_t *kp = st + ST_KF + 64 * tq;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 v = lds128(kp + 16 * q4);
                            bf[2 * q4][0] = v.x; bf[2 * q4][1] = v.y;
                            bf[2 * q4 + 1][0] = v.z; bf[2 * q4 + 1][1] = v.w;
                        }
                    }
                }
                if (FMT == DKV_FMT_FP16) {
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma16816(acc, qa[kk][0], 0u, qa[kk][1], 0u, bf[kk][0], bf[kk][1]);
                    x[nt][0] = acc[0];
                    x[nt][1] = acc[1];
                } else {
                    float acc[4][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                        mma16816(acc[j], qa[2 * j][0], 0u, qa[2 * j][1], 0u, bf[2 * j][0], bf[2 * j][1]);
                        mma16816(acc[j], qa[2 * j + 1][0], 0u, qa[2 * j + 1][1], 0u, bf[2 * j + 1][0],
                                 bf[2 * j + 1][1]);
                    }
                    // scales of positions 8nt + 2t + e
                    const int pa = 8 * nt + 2 * tq;
                    uint4 s0 = lds128(st + ST_SC + pa * SC_BYTES);
                    uint4 s1 = lds128(st + ST_SC + (pa + 1) * SC_BYTES);
                    if (first_seg && nt == 0 && tq == 0) {
                        // keyframe column: unit K weights; V weight 1 (SUFFIX) or 0 (PREFIX)
                        s0.x = s0.y = 0x3C003C00u;
                        s0.z = s0.w = (MODE == SUFFIX) ? 0x3C003C00u : 0u;
                    }
                    // slots past the end of the unit hold stale data: no V weight
                    if (pa >= npos) s0.z = s0.w = 0u;
                    if (pa + 1 >= npos) s1.z = s1.w = 0u;
                    x[nt][0] = acc[0][0] * h_lo(s0.x) + acc[1][0] * h_hi(s0.x) +
                               acc[2][0] * h_lo(s0.y) + acc[3][0] * h_hi(s0.y);
                    x[nt][1] = acc[0][1] * h_lo(s1.x) + acc[1][1] * h_hi(s1.x) +
                               acc[2][1] * h_lo(s1.y) + acc[3][1] * h_hi(s1.y);
                    dvh[nt][0][0] = s0.z; dvh[nt][0][1] = s0.w;
                    dvh[nt][1][0] = s1.z; dvh[nt][1][1] = s1.w;
                }
            }

            // ================= scores, online softmax =======================
            if (MODE != PLAIN) {
                quad_scan32(x, tq);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) { x[nt][0] += dot_carry; x[nt][1] += dot_carry; }
                dot_carry = __shfl_sync(0xffffffffu, x[3][1], 3, 4);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int slot = 8 * nt + 2 * tq + e;
                    const bool ok = head_ok && slot < npos;
                    x[nt][e] = ok ? x[nt][e] * A.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, x[nt][e]);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            const float alpha = exp2f(m_run - m_new);
            m_run = m_new;
            float psum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    x[nt][e] = exp2f(x[nt][e] - m_new);
                    psum += x[nt][e];
                }
            l_run = l_run * alpha + psum;

            // weights that multiply each position's dequantised row
            float wgt[4][2];
            if (MODE == SUFFIX) {
                float pin[4][2];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) { pin[nt][0] = x[nt][0]; pin[nt][1] = x[nt][1]; }
                const float tot = quad_scan32(pin, tq);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) wgt[nt][e] = tot - pin[nt][e] + x[nt][e];
            } else if (MODE == PREFIX) {
                e_carry *= alpha;
                float pin[4][2];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) { pin[nt][0] = x[nt][0]; pin[nt][1] = x[nt][1]; }
                const float tot = quad_scan32(pin, tq);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) wgt[nt][e] = -(e_carry + pin[nt][e] - x[nt][e]);
                e_carry += tot;
            } else {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) { wgt[nt][0] = x[nt][0]; wgt[nt][1] = x[nt][1]; }
            }

            // rescale the output accumulators (heads 2t, 2t+1 in the V layout)
            const float al0 = __shfl_sync(0xffffffffu, alpha, (2 * tq) * 4);
            const float al1 = __shfl_sync(0xffffffffu, alpha, (2 * tq + 1) * 4);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                o[mt][0] *= al0; o[mt][1] *= al1; o[mt][2] *= al0; o[mt][3] *= al1;
            }

            // ================= V side ======================================
            uint32_t vkf[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (FMT == DKV_FMT_DELTA && first_seg) {
                uint4 v0 = lds128(st + ST_KF + 256 + 32 * gq);
                uint4 v1 = lds128(st + ST_KF + 256 + 32 * gq + 16);
                vkf[0] = v0.x; vkf[1] = v0.y; vkf[2] = v0.z; vkf[3] = v0.w;
                vkf[4] = v1.x; vkf[5] = v1.y; vkf[6] = v1.z; vkf[7] = v1.w;
                if (MODE == PREFIX) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) vkf_keep[i] = vkf[i];
                }
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                // B' fragments: rows = positions 16kk + {2t,2t+1} | {2t+8, 2t+9}, col = head g
                // B' fragments: rows = positions 16kk + {2t,2t+1} | {2t+8, 2t+9}, col = head g.
                // For the delta format a weight multiplies a whole dequantised row
                // (the keyframe row, or a large delta) and its rounding is shared by
                // every channel, so it is carried as an fp16 hi + lo pair (about
                // 22 significant bits); the comparators weight one token per row and
                // use a single fp16 weight, as flash-decoding does.
                auto make_bp = [&](int j, uint32_t (&hi)[2], uint32_t (&lo)[2]) {
                    const int hw = j >> 1;
                    auto dv = [&](int nt, int e) {
                        uint32_t u = dvh[nt][e][hw];
                        return (j & 1) ? h_hi(u) : h_lo(u);
                    };
                    const float v0 = wgt[2 * kk][0] * dv(2 * kk, 0);
                    const float v1 = wgt[2 * kk][1] * dv(2 * kk, 1);
                    const float v2 = wgt[2 * kk + 1][0] * dv(2 * kk + 1, 0);
                    const float v3 = wgt[2 * kk + 1][1] * dv(2 * kk + 1, 1);
                    hi[0] = pack_h2(v0, v1);
                    hi[1] = pack_h2(v2, v3);
                    if (FMT == DKV_FMT_DELTA) {
                        lo[0] = pack_h2(v0 - h_lo(hi[0]), v1 - h_hi(hi[0]));
                        lo[1] = pack_h2(v2 - h_lo(hi[1]), v3 - h_hi(hi[1]));
                    }
                };
                uint32_t bp[2] = {0u, 0u}, bl[2] = {0u, 0u};
                if (FMT == DKV_FMT_FP16) {
                    bp[0] = pack_h2(wgt[2 * kk][0], wgt[2 * kk][1]);
                    bp[1] = pack_h2(wgt[2 * kk + 1][0], wgt[2 * kk + 1][1]);
                }
                const int sA = 16 * kk + 2 * tq;
                if (FMT == DKV_FMT_FP16) {
                    const uint8_t *vb = st + 8192 + 32 * gq;
                    uint4 A0 = lds128(vb + sA * 256), A1 = lds128(vb + sA * 256 + 16);
                    uint4 B0 = lds128(vb + (sA + 1) * 256), B1 = lds128(vb + (sA + 1) * 256 + 16);
                    uint4 C0 = lds128(vb + (sA + 8) * 256), C1 = lds128(vb + (sA + 8) * 256 + 16);
                    uint4 D0 = lds128(vb + (sA + 9) * 256), D1 = lds128(vb + (sA + 9) * 256 + 16);
                    uint32_t wa[8] = {A0.x, A0.y, A0.z, A0.w, A1.x, A1.y, A1.z, A1.w};
                    uint32_t wb[8] = {B0.x, B0.y, B0.z, B0.w, B1.x, B1.y, B1.z, B1.w};
                    uint32_t wc[8] = {C0.x, C0.y, C0.z, C0.w, C1.x, C1.y, C1.z, C1.w};
                    uint32_t wd[8] = {D0.x, D0.y, D0.z, D0.w, D1.x, D1.y, D1.z, D1.w};
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        const uint32_t a0 = prmt(wa[mt], wb[mt], 0x5410u);
                        const uint32_t a1 = prmt(wa[mt], wb[mt], 0x7632u);
                        const uint32_t a2 = prmt(wc[mt], wd[mt], 0x5410u);
                        const uint32_t a3 = prmt(wc[mt], wd[mt], 0x7632u);
                        mma16816(o[mt], a0, a1, a2, a3, bp[0], bp[1]);
                    }
                } else {
                    const uint8_t *vb = st + ST_VN + 8 * gq;
                    const uint2 wA = lds64(vb + sA * NIB_BYTES);
                    const uint2 wB = lds64(vb + (sA + 1) * NIB_BYTES);
                    const uint2 wC = lds64(vb + (sA + 8) * NIB_BYTES);
                    const uint2 wD = lds64(vb + (sA + 9) * NIB_BYTES);
                    const bool kfrow = (FMT == DKV_FMT_DELTA) && (MODE == SUFFIX) && first_seg &&
                                       kk == 0 && tq == 0;
                    const uint32_t sel0 = kfrow ? 0x3254u : 0x3210u;
                    const uint32_t sel1 = kfrow ? 0x3276u : 0x3210u;
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        const int i = mt & 3;
                        const uint32_t sel = (uint32_t)(i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12));
                        const uint32_t m01 = prmt(mt < 4 ? wA.x : wA.y, mt < 4 ? wB.x : wB.y, sel);
                        const uint32_t m23 = prmt(mt < 4 ? wC.x : wC.y, mt < 4 ? wD.x : wD.y, sel);
                        uint32_t a0, a1, a2, a3;
                        {
                            const uint32_t MAGIC = 0x64006400u;
                            const __half2 SUB_LO = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
                            const __half2 MUL_HI = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
                            const __half2 SUB_HI = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
                            a0 = h2_as_u32(__hsub2(u32_as_h2(lop_and_or(m01, 0x000F000Fu, MAGIC)), SUB_LO));
                            a1 = h2_as_u32(__hfma2(u32_as_h2(lop_and_or(m01, 0x00F000F0u, MAGIC)), MUL_HI, SUB_HI));
                            a2 = h2_as_u32(__hsub2(u32_as_h2(lop_and_or(m23, 0x000F000Fu, MAGIC)), SUB_LO));
                            a3 = h2_as_u32(__hfma2(u32_as_h2(lop_and_or(m23, 0x00F000F0u, MAGIC)), MUL_HI, SUB_HI));
                        }
                        if (FMT == DKV_FMT_DELTA && MODE == SUFFIX && kk == 0) {
                            a0 = prmt(a0, vkf[mt], sel0);
                            a1 = prmt(a1, vkf[mt], sel1);
                        }
                        const int j = mt >> 1;
                        if ((mt & 1) == 0) make_bp(j, bp, bl);
                        mma16816(o[mt], a0, a1, a2, a3, bp[0], bp[1]);
                        if (FMT == DKV_FMT_DELTA) mma16816(o[mt], a0, a1, a2, a3, bl[0], bl[1]);
                        if (MODE == PREFIX) {
                            // R += sum_s (code-8) * d_s : B = the scales alone
                            uint32_t r0, r1;
                            {
                                const int hw = j >> 1;
                                auto dv = [&](int nt, int e) {
                                    uint32_t u = dvh[nt][e][hw];
                                    return (j & 1) ? h_hi(u) : h_lo(u);
                                };
                                r0 = pack_h2(dv(2 * kk, 0), dv(2 * kk, 1));
                                r1 = pack_h2(dv(2 * kk + 1, 0), dv(2 * kk + 1, 1));
                            }
                            mma16816(racc[mt], a0, a1, a2, a3, r0, r1);
                        }
                    }
                }
            }

            // PREFIX: close the group  o += W_g (v_f + R_g)
            if (MODE == PREFIX && last_seg) {
                const float w0 = __shfl_sync(0xffffffffu, e_carry, (2 * tq) * 4);
                const float w1 = __shfl_sync(0xffffffffu, e_carry, (2 * tq + 1) * 4);
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const float v_lo = h_lo(vkf_keep[mt]) + racc[mt][0];   // channel 16mt+g
                    const float v_hi = h_hi(vkf_keep[mt]) + racc[mt][2];   // channel 16mt+g+8
                    o[mt][0] += w0 * v_lo; o[mt][1] += w1 * v_lo;
                    o[mt][2] += w0 * v_hi; o[mt][3] += w1 * v_hi;
                    racc[mt][0] = racc[mt][1] = racc[mt][2] = racc[mt][3] = 0.f;
                }
                e_carry = 0.f;
                dot_carry = 0.f;
            } else if (MODE == SUFFIX) {
                dot_carry = 0.f;
            }
        }

        // ---- release the stage and refill it ------------------------------
        __syncwarp();
        if (ic.valid()) {
            if (lane == 0 && !dead) {
                fence_proxy_async();
                issue_stage<FMT>(cv, ic, nvs_per_kv, mystages + stage_i * STAGE, mybar + stage_i);
            }
            cursor_next(ic, cv, nvs);
        }
        stage_i = (stage_i + 1 == NS) ? 0 : stage_i + 1;
        cursor_next(cc, cv, nvs);
    }
    if (cur_b >= 0) flush();

    // A warp that gave up still owns copies in flight: wait for them (bounded)
    // before the CTA can exit and its shared memory be reused.
    if (dead) {
        for (int s = 0; s < NS; ++s) {
            if (lane == 0) (void)mbar_wait_bounded(mybar + s, (phase >> s) & 1);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// merge: grid (Hq, B), 128 threads (one per channel)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) merge_kernel(CacheView cv, int Hq, int G, int NHG,
                                                    int64_t NW, const float *ws, float *out) {
    const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
    const int nvs = cv.Hkv * NHG;
    __shared__ int64_t sh_plan[2];
    __shared__ int64_t sh_total;
    if (threadIdx.x == 0) {
        int64_t acc = 0, mine = 0;
        for (int bb = 0; bb < cv.B; ++bb) {
            if (bb == b) mine = acc;
            int l = cv.seqlen[bb];
            if (l < 0 || l > cv.cap) l = 0;
            acc += (int64_t)nvs * units_of(cv.fmt, cv.kf, l);
        }
        sh_plan[0] = mine;
        sh_total = acc;
    }
    __syncthreads();
    int len = cv.seqlen[b];
    if (len < 0 || len > cv.cap) len = 0;
    const int ub = units_of(cv.fmt, cv.kf, len);
    float *dst = out + ((int64_t)b * Hq + h) * D;
    if (ub == 0) { dst[c] = 0.f; return; }
    const int kvh = h / G, hl = h % G, hg = hl >> 3, j = hl & 7;
    const int vsl = kvh * NHG + hg;
    const int64_t vseq = (int64_t)b * nvs + vsl;
    const int64_t T = sh_total;
    const int64_t xs = sh_plan[0] + (int64_t)vsl * ub, xe = xs + ub;
    const int64_t w0 = warp_of(xs, NW, T), w1 = warp_of(xe - 1, NW, T);
    float M = -INFINITY;
    for (int64_t w = w0; w <= w1; ++w) {
        if (range_start(w, NW, T) >= range_start(w + 1, NW, T)) continue;
        M = fmaxf(M, ws[(w + vseq) * PARTIAL_FLOATS + j]);
    }
    float L = 0.f, O = 0.f;
    for (int64_t w = w0; w <= w1; ++w) {
        if (range_start(w, NW, T) >= range_start(w + 1, NW, T)) continue;
        const float *rec = ws + (w + vseq) * PARTIAL_FLOATS;
        const float sc = exp2f(rec[j] - M);
        L += rec[8 + j] * sc;
        O += rec[16 + j * 128 + c] * sc;
    }
    dst[c] = O / L;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int FMT, int MODE>
static size_t split_smem() {
    using Cfg = FmtCfg<FMT>;
    return 8 * (MAX_B + 1) + 8 * WARPS * Cfg::NS + 64 + 128 + (size_t)WARPS * Cfg::NS * Cfg::STAGE;
}

template <int FMT, int MODE>
static cudaError_t geom_for(SplitGeom *g) {
    static int cached_dev = -1, cached_ctas = 0;
    int dev;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev != cached_dev) {
        const size_t sm = split_smem<FMT, MODE>();
        e = cudaFuncSetAttribute(split_kernel<FMT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sm);
        if (e != cudaSuccess) return e;
        int per_sm = 0, nsm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, split_kernel<FMT, MODE>,
                                                          WARPS * 32, sm);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        cached_ctas = (per_sm < 1 ? 1 : per_sm) * nsm;
        cached_dev = dev;
    }
    g->ctas = cached_ctas;
    g->warps_per_cta = WARPS;
    return cudaSuccess;
}

cudaError_t split_geometry(int fmt, int kf, int batch, SplitGeom *g) {
    (void)batch;
    if (fmt == DKV_FMT_DELTA) {
        return kf <= SEG ? geom_for<DKV_FMT_DELTA, SUFFIX>(g) : geom_for<DKV_FMT_DELTA, PREFIX>(g);
    }
    if (fmt == DKV_FMT_Q4_0) return geom_for<DKV_FMT_Q4_0, PLAIN>(g);
    return geom_for<DKV_FMT_FP16, PLAIN>(g);
}

template <int FMT, int MODE>
static cudaError_t launch_split_t(const SplitArgs &a, cudaStream_t st) {
    SplitGeom g;
    cudaError_t e = geom_for<FMT, MODE>(&g);
    if (e != cudaSuccess) return e;
    split_kernel<FMT, MODE><<<g.ctas, WARPS * 32, split_smem<FMT, MODE>(), st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_split(const CacheView &cv, const void *Q, int q_dtype, int Hq,
                         float softmax_scale, float *ws, int64_t ws_floats, cudaStream_t st) {
    (void)ws_floats;
    SplitArgs a;
    a.cv = cv;
    a.Q = Q;
    a.q_dtype = q_dtype;
    a.Hq = Hq;
    a.G = Hq / cv.Hkv;
    a.NHG = (a.G + 7) / 8;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.ws = ws;
    if (cv.fmt == DKV_FMT_DELTA) {
        return cv.kf <= SEG ? launch_split_t<DKV_FMT_DELTA, SUFFIX>(a, st)
                            : launch_split_t<DKV_FMT_DELTA, PREFIX>(a, st);
    }
    if (cv.fmt == DKV_FMT_Q4_0) return launch_split_t<DKV_FMT_Q4_0, PLAIN>(a, st);
    return launch_split_t<DKV_FMT_FP16, PLAIN>(a, st);
}

cudaError_t launch_merge(const CacheView &cv, int Hq, float *out, const float *ws, cudaStream_t st) {
    SplitGeom g;
    cudaError_t e = split_geometry(cv.fmt, cv.kf, cv.B, &g);
    if (e != cudaSuccess) return e;
    const int G = Hq / cv.Hkv;
    const int NHG = (G + 7) / 8;
    dim3 grid(Hq, cv.B);
    merge_kernel<<<grid, 128, 0, st>>>(cv, Hq, G, NHG, (int64_t)g.ctas * g.warps_per_cta, ws, out);
    return cudaGetLastError();
}

}  // namespace dkv
