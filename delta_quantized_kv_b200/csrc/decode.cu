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
//   K side  D[p][h] = sum_c code[p][c] * q[h][c]  per 32-channel block, m16n8k16
//           with positions as M, channels as K and heads as N (q stays in
//           registers as the B operand);
//   V side  O[c][h] += sum_p code[p][c] * (S[h][p] * d[p][blk(c)]), m16n8k16
//           with channels as M, positions as K and heads as N.
// An 8x8 movmatrix transpose turns the K-side accumulator layout (a thread
// owns positions x heads 2t, 2t+1) into the V-side B fragments.
//
// Groups longer than one 32-position stage (kf > 32) use the equivalent
// forward form  sum_p w_p v^_p = W_g (v_f + R_g) - sum_s delta^_s E_s  with
// E_s the exclusive prefix of the weights inside the group and R_g the sum of
// the group's dequantised deltas (an extra MMA against the scales alone).
//
// Work split: the (sequence, unit) pairs of all sequences are flattened and
// cut into equal contiguous ranges, one per warp of a persistent grid.  Each
// warp streams its range through its own ring of shared-memory stages filled
// by 1-D bulk async copies (cp.async.bulk + mbarrier), keeps an online-softmax
// state per sequence it touches, and writes one partial (max, sum, output)
// record per such sequence.  The merge kernel combines the partial records
// with a log-sum-exp.
#include <atomic>
#include <cstdint>
#include <mutex>

#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace dkv {

enum Mode { SUFFIX = 0, PREFIX = 1, PLAIN = 2 };

#ifndef DKV_WARPS
#define DKV_WARPS 4
#endif
constexpr int WARPS = DKV_WARPS;             // warps per CTA (independent pipelines)

// Nibble formats with kf <= 32: units per stage, stages per warp, CTAs per SM.
// Two groups per stage and one stage per warp (a warp's next stage is copied
// while the other warps of the SM compute) measured fastest on B200: the
// shared memory this frees buys a third CTA per SM.
#ifndef DKV_PFX_NU
#define DKV_PFX_NU 2             // kf > 32: consecutive segments of one group per stage
#endif
#ifndef DKV_PFX_MINB
#define DKV_PFX_MINB 3           // kf > 32: CTAs per SM the registers are sized for
#endif
#ifndef DKV_QSM
#define DKV_QSM 1                // q fragments in shared memory (0: registers)
#endif
#ifndef DKV_MERGE_BATCH
#define DKV_MERGE_BATCH 4        // partial records a merge warp loads per round trip
#endif
#ifndef DKV_NIB_NU
#define DKV_NIB_NU 2
#endif
#ifndef DKV_NIB_NS
#define DKV_NIB_NS 1
#endif
#ifndef DKV_NIB_MINB
#define DKV_NIB_MINB 3
#endif

// Per (format, mode): units per stage, stage bytes, stages per warp, CTAs/SM.
// A unit is one keyframe group (delta, kf <= 32), one 32-position segment of
// a group (delta, kf > 32), or one 32-position chunk (Q4_0, fp16).
template <int FMT, int MODE> struct KCfg {
    static constexpr bool NIB = FMT != DKV_FMT_FP16 && MODE != PREFIX;
    static constexpr int NU = NIB ? DKV_NIB_NU : (MODE == PREFIX ? DKV_PFX_NU : 1);
    static constexpr int STAGE = FMT == DKV_FMT_FP16 ? 16384 : NU * 5120;
    static constexpr int NS = NIB ? DKV_NIB_NS : (MODE == PREFIX && NU == 2 ? 1 : 2);
    static constexpr int MINB = FMT == DKV_FMT_FP16 ? 1 : (MODE == PREFIX ? DKV_PFX_MINB : DKV_NIB_MINB);
};

// Shared-memory map of the split kernel: [mbarriers WARPS*NS x 8 B]
// [stage descriptors WARPS*NS x 16 B][stages WARPS*NS x STAGE], each region
// aligned; the offsets follow from NS so no region can overlap another.
template <int FMT, int MODE> struct SmemMap {
    static constexpr int NS = KCfg<FMT, MODE>::NS, STAGE = KCfg<FMT, MODE>::STAGE;
    static constexpr int BAR_OFF = 0;
    static constexpr int META_OFF = ((BAR_OFF + 8 * WARPS * NS) + 15) / 16 * 16;
    static constexpr int STAGE_OFF = ((META_OFF + 32 * WARPS * NS) + 127) / 128 * 128;
    static constexpr int Q_OFF = STAGE_OFF + WARPS * NS * STAGE;       // q fragments (DKV_QSM)
    static constexpr int BYTES = Q_OFF + (DKV_QSM ? WARPS * 2048 : 0);
    static_assert(META_OFF >= BAR_OFF + 8 * WARPS * NS, "barriers overlap descriptors");
    static_assert(STAGE_OFF >= META_OFF + 32 * WARPS * NS, "descriptors overlap stages");
    static_assert(STAGE % 128 == 0, "stages must stay 128-byte aligned");
    static_assert(BYTES <= 227 * 1024, "shared memory per CTA");
};


// Work units of a sequence of len tokens: keyframe groups for the delta
// format with kf <= 32; 32-position segments of the groups for kf > 32 (a
// group of kf tokens holds ceil(kf / 32) of them); 32-position chunks for the
// comparators.
__host__ __device__ inline int seg_per_group(int kf) { return (kf + SEG - 1) / SEG; }
__host__ __device__ inline int units_of(int fmt, int kf, int len) {
    if (len <= 0) return 0;
    if (fmt != DKV_FMT_DELTA) return (len + SEG - 1) / SEG;
    if (kf <= SEG) return (len + kf - 1) / kf;
    return (len / kf) * seg_per_group(kf) + (len % kf + SEG - 1) / SEG;
}
// First position of unit u of a sequence (units are contiguous in position).
__host__ __device__ inline int64_t unit_pos(int fmt, int kf, int64_t u) {
    if (fmt != DKV_FMT_DELTA) return u * SEG;
    if (kf <= SEG) return u * kf;
    const int spg = seg_per_group(kf);
    return (u / spg) * kf + (u % spg) * SEG;
}

// Warp w of NW owns units [w*T/NW, (w+1)*T/NW).
__host__ __device__ inline int64_t range_start(int64_t w, int64_t NW, int64_t T) {
    return (w * T) / NW;
}
__host__ __device__ inline int64_t warp_of(int64_t x, int64_t NW, int64_t T) {
    return ((x + 1) * NW - 1) / T;
}

struct SplitArgs {
    CacheView cv;
    const void *Q;
    int q_dtype;
    int Hq, G, NHG;            // query heads, heads per kv head, head groups of 8
    int nq;                    // queries per sequence (the newest nq tokens' own, causal)
    float scale_log2;          // softmax_scale * log2(e), > 0
    float wshift;              // log2 of the factor every softmax weight is scaled down by
    float *ws;                 // partial records
    int64_t ws_floats;         // workspace size (checked builds test every record against it)
    float *heads, *hands;      // kf > 32: the records of groups entered midway, the handoffs
    int fault;                 // test support: 1 = arm the copy barriers but issue no copy
    // fused append (cv.len_add = n > 0): the n new tokens of each sequence,
    // [B][Hkv][n][D] of kv_dtype
    const void *Kn, *Vn;
    int kv_dtype;
};

// Stored length of batch entry b, and whether the entry takes the call's new
// tokens (fused append): its length is valid and the tokens fit.
__device__ inline bool takes_append(const CacheView &cv, int b, int &l) {
    l = cv.seqlen[b];
    return l >= 0 && l <= cv.cap && l + cv.len_add <= cv.cap;
}

// Length decoded for batch entry b: 0 for an invalid stored length; with a
// fused append, the stored length plus the new tokens when they fit.
__device__ inline int clamp_len(const CacheView &cv, int b) {
    int l = cv.seqlen[b];
    if (l < 0 || l > cv.cap) return 0;
    return l + cv.len_add <= cv.cap ? l + cv.len_add : l;
}

// Iterates the (unit, segment) stage items of one warp's range in order.
struct Cursor {
    int64_t left;              // units left in the range, the current one included
    int b, vs, g;              // batch entry, sequence within the batch entry, group / chunk
    int units_b;               // units per sequence of batch entry b
    int groups_b;              // values of g per sequence of batch entry b
    int len_b;                 // tokens of batch entry b
    int seg, nseg;             // segment within group g and the group's segments (kf > 32)
    bool head;                 // kf > 32: group g was entered after its first segment
    const uint8_t *seq;        // data of sequence (b, kv head of vs) (contiguous caches)
    // paged caches, issuing lane only: the page last looked up
    int pb, pv, pidx;          // its batch entry, sequence and block-table column
    const uint8_t *pbase;      // its records of kv head vs / nhg (null: entry was bad)
    __device__ bool valid() const { return left > 0; }
};

template <int MODE>
__device__ inline int nseg_of(const CacheView &cv, int len, int g) {
    if (MODE != PREFIX) return 1;
    const int glen = min(cv.kf, len - g * cv.kf);
    return (glen + SEG - 1) / SEG;
}

// Warp-wide: total units over all batch entries, and (if 0 <= r < total) the
// batch entry b containing unit r with the index of its first unit.
__device__ inline int64_t locate(const CacheView &cv, int nvs, int64_t r, int &b_out,
                                 int64_t &base_out) {
    const int lane = threadIdx.x & 31;
    int64_t base = 0;
    b_out = -1;
    base_out = 0;
    for (int b0 = 0; b0 < cv.B; b0 += 32) {
        const int b = b0 + lane;
        const int64_t u = b < cv.B ? (int64_t)nvs * units_of(cv.fmt, cv.kf, clamp_len(cv, b)) : 0;
        int64_t inc = u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        const int64_t chunk = __shfl_sync(0xffffffffu, inc, 31);
        if (b_out < 0 && r >= base && r < base + chunk) {
            const unsigned m = __ballot_sync(0xffffffffu, base + inc > r);
            const int l = __ffs(m) - 1;
            b_out = b0 + l;
            base_out = base + __shfl_sync(0xffffffffu, inc - u, l);
        }
        base += chunk;
    }
    return base;
}

__device__ inline const uint8_t *seq_ptr(const CacheView &cv, int b, int vs, int nhg) {
    const int kvh = nhg == 1 ? vs : vs / nhg;
    return cv.data + ((int64_t)b * cv.Hkv + kvh) * cv.seq_stride;
}

template <int MODE>
__device__ inline void cursor_seek(Cursor &c, const CacheView &cv, int nvs, int nhg, int64_t x,
                                   int64_t count) {
    int b;
    int64_t base;
    locate(cv, nvs, x, b, base);
    c.left = count;
    c.b = b;
    c.len_b = clamp_len(cv, b);
    c.units_b = units_of(cv.fmt, cv.kf, c.len_b);
    const int64_t r = x - base;
    c.vs = (int)(r / c.units_b);
    const int u = (int)(r % c.units_b);
    if (MODE == PREFIX) {
        const int spg = seg_per_group(cv.kf);
        c.groups_b = (c.len_b + cv.kf - 1) / cv.kf;
        c.g = u / spg;
        c.seg = u % spg;
        c.head = c.seg != 0;
    } else {
        c.groups_b = c.units_b;
        c.g = u;
        c.seg = 0;
        c.head = false;
    }
    c.nseg = nseg_of<MODE>(cv, c.len_b, c.g);
    c.seq = seq_ptr(cv, c.b, c.vs, nhg);
    c.pb = -1;
}

template <int MODE>
__device__ inline void cursor_next(Cursor &c, const CacheView &cv, int nvs, int nhg) {
    if (--c.left == 0) return;
    if (MODE == PREFIX && ++c.seg < c.nseg) return;
    c.seg = 0;
    c.head = false;
    if (++c.g == c.groups_b) {
        c.g = 0;
        if (++c.vs == nvs) {
            c.vs = 0;
            do {
                ++c.b;
                c.len_b = clamp_len(cv, c.b);
                c.units_b = units_of(cv.fmt, cv.kf, c.len_b);
            } while (c.units_b == 0);
            c.groups_b = MODE == PREFIX ? (c.len_b + cv.kf - 1) / cv.kf : c.units_b;
        }
        c.seq = seq_ptr(cv, c.b, c.vs, nhg);
    }
    if (MODE == PREFIX) c.nseg = nseg_of<MODE>(cv, c.len_b, c.g);
}

// Fused append: the lengths the split kernel decoded, int32[B], after the
// partial records of the workspace (NW warp slots + one per sequence).
__host__ __device__ inline int32_t *merge_lengths(float *ws, int64_t NW, int64_t nseq) {
    return reinterpret_cast<int32_t *>(ws + (NW + nseq) * PARTIAL_FLOATS);
}
// kf > 32, after the lengths: per warp slot, the partial record of the group
// its range entered after the group's first segment (scores relative to the
// state before its first position); then the log2 softmax scale (a header of
// HAND_HDR floats) and, per warp slot, the state it hands to the next warp
// when its range ends inside a group: the dot of each head's query with the
// reconstructed key of its last position (8 floats) and the reconstructed
// value row there (128 floats).  Both are relative to the state the warp
// entered the group with when it entered it after the first segment,
// absolute otherwise.
__host__ __device__ inline float *head_records(float *ws, int64_t NW, int64_t nseq, int B) {
    return ws + (NW + nseq) * PARTIAL_FLOATS + ((int64_t)B + 3) / 4 * 4;
}
__host__ __device__ inline float *handoffs(float *ws, int64_t NW, int64_t nseq, int B) {
    return head_records(ws, NW, nseq, B) + NW * PARTIAL_FLOATS;
}

// What the consumer needs to know about a stage, written next to the stage by
// the issuing lane before it arms the barrier.
struct StageMeta {
    int b, vs;                 // batch entry, sequence within it
    int npos;                  // valid positions: unit 0 in bits 0-7, unit 1 in bits 8-15
    int flags;                 // kf > 32: the STG_* bits below
    int pos0;                  // position of unit 0's first slot in its sequence
    int pad[3];
};
static_assert(sizeof(StageMeta) == 32, "stage descriptors are 32 bytes");
// Stage flags (kf > 32: one or two segments of one group per stage).
constexpr int STG_FIRST = 1;   // first segment of its group: slot 0 is the keyframe
constexpr int STG_CLOSE = 2;   // the group's last segment in this warp's range
constexpr int STG_HEAD = 4;    // the range entered this group after its first segment
constexpr int STG_HAND = 8;    // the range ends inside this group (hand the state on)

// Positions of the current unit of c.
__device__ inline int unit_npos(const CacheView &cv, const Cursor &c, int g) {
    if (cv.fmt == DKV_FMT_DELTA) {
        const int glen = min(cv.kf, c.len_b - g * cv.kf);
        return min(SEG, glen - c.seg * SEG);
    }
    return min(SEG, c.len_b - g * SEG);
}

// Stage layouts in shared memory (offsets from the stage start), unit u:
//  DELTA, kf <= 32: NU consecutive group records copied as one run, record u
//      at u * rec: [K kf 256][V kf 256][scales (kf-1)x16][K nib (kf-1)x64]
//      [V nib (kf-1)x64];
//  DELTA, kf > 32 (NU consecutive 32-position segments of one group):
//      [K kf 256][V kf 256][scales NU*32 x16][K nib NU*32 x64][V nib NU*32 x64];
//  Q4_0 (NU chunks of 32 positions): [scales NU x 512][K nib NU x 2048]
//      [V nib NU x 2048];
//  FP16 (NU = 1): [K 32x256][V 32x256].
// For slot s (position a + s) the scale / K nibble / V nibble rows start at
// sc0 + 16 s, kn0 + 64 s, vn0 + 64 s; keyframes at kf0 (K) and kf0 + 256 (V).
struct StageMap {
    int kf0, sc0, kn0, vk0, vn0;
};
template <int FMT, int MODE>
__device__ inline StageMap stage_map(int kf, int64_t rec, int u) {
    constexpr int NU = KCfg<FMT, MODE>::NU;
    StageMap m;
    if (FMT == DKV_FMT_DELTA && MODE == SUFFIX) {
        const int base = u * (int)rec;
        m.kf0 = base;
        m.sc0 = base + KF_BYTES - SC_BYTES;
        m.kn0 = base + KF_BYTES + (kf - 1) * SC_BYTES - NIB_BYTES;
        m.vk0 = base + 256;
        m.vn0 = base + KF_BYTES + (kf - 1) * (SC_BYTES + NIB_BYTES) - NIB_BYTES;
    } else if (FMT == DKV_FMT_DELTA) {
        m.kf0 = 0;
        m.vk0 = 256;
        m.sc0 = 512 + 512 * u;
        m.kn0 = 512 + 512 * NU + 2048 * u;
        m.vn0 = 512 + 2560 * NU + 2048 * u;
    } else if (FMT == DKV_FMT_Q4_0) {
        m.kf0 = 0;
        m.sc0 = 512 * u;
        m.kn0 = 512 * NU + 2048 * u;
        m.vk0 = 256;
        m.vn0 = 2560 * NU + 2048 * u;
    } else {
        m.kf0 = 0;
        m.sc0 = 512;
        m.kn0 = 1024;
        m.vk0 = 256;
        m.vn0 = 3072;
    }
    return m;
}

// First record of the cursor's current unit (delta format).  Paged: the
// block table is read once per page (the issuing lane keeps the page's base).
template <bool PAGED>
__device__ inline const uint8_t *stage_rec(const CacheView &cv, Cursor &c, int nhg) {
    if (!PAGED) return c.seq + (int64_t)c.g * cv.rec_bytes;
    const int pidx = c.g / cv.pg;
    if (c.pb != c.b || c.pv != c.vs || c.pidx != pidx) {
        const int kvh = nhg == 1 ? c.vs : c.vs / nhg;
        c.pbase = rec_ptr<true>(cv, c.b, kvh, pidx * cv.pg);
        c.pb = c.b;
        c.pv = c.vs;
        c.pidx = pidx;
    }
    return c.pbase ? c.pbase + (int64_t)(c.g - pidx * cv.pg) * cv.rec_bytes : nullptr;
}

// Issue the bulk copies of one stage (nu units starting at c; one lane).
template <int FMT, int MODE, bool PAGED>
__device__ inline void issue_stage(const CacheView &cv, Cursor &c, int nhg, int nu,
                                   int npos_all, uint8_t *stage, uint64_t *bar, int fault) {
    constexpr int NU = KCfg<FMT, MODE>::NU, STAGE = KCfg<FMT, MODE>::STAGE;
    const uint8_t *sb = c.seq;
    if (fault) {
        // test support: expect bytes that never come, so the consumer's bounded
        // wait runs out and reports DKV_DEV_TIMEOUT
        mbar_arrive_expect_tx(bar, 16);
        return;
    }
    if (FMT == DKV_FMT_DELTA && MODE == SUFFIX) {
        // nu consecutive records (one page holds both when paged)
        const uint8_t *rec = stage_rec<PAGED>(cv, c, nhg);
        if (!rec) {                      // bad block-table entry: flagged, nothing copied
            mbar_arrive_expect_tx(bar, 0);
            return;
        }
        const uint32_t bytes = (uint32_t)(nu * cv.rec_bytes);
        if (!rec_ok(cv, rec, bytes) || !range_ok(cv.header, stage, bytes, stage, STAGE)) {
            mbar_arrive_expect_tx(bar, 0);   // checked build: nothing copied
            return;
        }
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(stage, rec, bytes, bar);
    } else if (FMT == DKV_FMT_DELTA) {
        // nu consecutive segments of group c.g from segment c.seg on
        const int kf = cv.kf;
        const int a = c.seg * SEG;
        const int npos = npos_all;
        const uint8_t *rec = stage_rec<PAGED>(cv, c, nhg);
        if (!rec) {
            mbar_arrive_expect_tx(bar, 0);
            return;
        }
        const uint8_t *scs = rec + KF_BYTES;
        const uint8_t *kns = scs + (int64_t)(kf - 1) * SC_BYTES;
        const uint8_t *vns = kns + (int64_t)(kf - 1) * NIB_BYTES;
        // slot s of the stage holds position a + s, i.e. delta index a + s - 1
        const int s0 = (a == 0) ? 1 : 0;       // slot 0 of segment 0 is the keyframe
        const int nd = npos - s0;
        const int di0 = a + s0 - 1;
        const uint32_t bytes = (a == 0 ? KF_BYTES : 0) + nd * (SC_BYTES + 2 * NIB_BYTES);
        const StageMap sm = stage_map<FMT, MODE>(kf, cv.rec_bytes, 0);
        if (DKV_CHECKED &&
            !(rec_ok(cv, rec, (int64_t)cv.rec_bytes) &&
              rec_ok(cv, scs + (int64_t)di0 * SC_BYTES, (int64_t)nd * SC_BYTES) &&
              rec_ok(cv, kns + (int64_t)di0 * NIB_BYTES, (int64_t)nd * NIB_BYTES) &&
              rec_ok(cv, vns + (int64_t)di0 * NIB_BYTES, (int64_t)nd * NIB_BYTES) &&
              range_ok(cv.header, stage + sm.vn0 + s0 * NIB_BYTES, (int64_t)nd * NIB_BYTES, stage,
                       STAGE))) {
            mbar_arrive_expect_tx(bar, 0);   // checked build: nothing copied
            return;
        }
        mbar_arrive_expect_tx(bar, bytes);
        if (a == 0) bulk_g2s(stage, rec, KF_BYTES, bar);
        if (nd > 0) {
            bulk_g2s(stage + sm.sc0 + s0 * SC_BYTES, scs + (int64_t)di0 * SC_BYTES, nd * SC_BYTES,
                     bar);
            bulk_g2s(stage + sm.kn0 + s0 * NIB_BYTES, kns + (int64_t)di0 * NIB_BYTES,
                     nd * NIB_BYTES, bar);
            bulk_g2s(stage + sm.vn0 + s0 * NIB_BYTES, vns + (int64_t)di0 * NIB_BYTES,
                     nd * NIB_BYTES, bar);
        }
    } else if (FMT == DKV_FMT_Q4_0) {
        const int p0 = c.g * SEG;
        if (!rec_ok(cv, sb + (int64_t)p0 * SC_BYTES, (int64_t)npos_all * SC_BYTES) ||
            !rec_ok(cv, sb + (int64_t)cv.cap * (SC_BYTES + NIB_BYTES) + (int64_t)p0 * NIB_BYTES,
                    (int64_t)npos_all * NIB_BYTES)) {
            mbar_arrive_expect_tx(bar, 0);   // checked build: nothing copied
            return;
        }
        mbar_arrive_expect_tx(bar, npos_all * (SC_BYTES + 2 * NIB_BYTES));
        bulk_g2s(stage, sb + (int64_t)p0 * SC_BYTES, npos_all * SC_BYTES, bar);
        bulk_g2s(stage + 512 * NU, sb + (int64_t)cv.cap * SC_BYTES + (int64_t)p0 * NIB_BYTES,
                 npos_all * NIB_BYTES, bar);
        bulk_g2s(stage + 2560 * NU, sb + (int64_t)cv.cap * (SC_BYTES + NIB_BYTES) + (int64_t)p0 * NIB_BYTES,
                 npos_all * NIB_BYTES, bar);
    } else {
        const int p0 = c.g * SEG;
        if (!rec_ok(cv, sb + (int64_t)p0 * 256, (int64_t)npos_all * 256) ||
            !rec_ok(cv, sb + (int64_t)cv.cap * 256 + (int64_t)p0 * 256, (int64_t)npos_all * 256)) {
            mbar_arrive_expect_tx(bar, 0);   // checked build: nothing copied
            return;
        }
        mbar_arrive_expect_tx(bar, npos_all * 512);
        bulk_g2s(stage, sb + (int64_t)p0 * 256, npos_all * 256, bar);
        bulk_g2s(stage + 8192, sb + (int64_t)cv.cap * 256 + (int64_t)p0 * 256, npos_all * 256, bar);
    }
}

// Decide how many units the next stage takes (the units must be consecutive
// in one sequence), fill its descriptor and (lane 0) issue its copies; every
// lane advances its cursor identically.
// With one stage per warp the descriptor stays in registers (every lane
// computes it); with more it goes to the stage's shared-memory slot.
template <int FMT, int MODE, bool PAGED>
__device__ inline StageMeta next_stage(const CacheView &cv, Cursor &c, int nvs, int nhg,
                                       uint8_t *stage, uint64_t *bar, StageMeta *meta, int lane,
                                       int fault) {
    constexpr int NU = KCfg<FMT, MODE>::NU;
    const int np0 = unit_npos(cv, c, c.g);
    int nu = 1, np1 = 0;
    if (MODE == PREFIX) {
        // two consecutive segments of one group per stage
        if (NU == 2 && c.left >= 2 && c.seg + 1 < c.nseg) {
            nu = 2;
            np1 = min(SEG, min(cv.kf, c.len_b - c.g * cv.kf) - (c.seg + 1) * SEG);
        }
    } else if (NU == 2 && c.left >= 2 && c.g + 1 < c.units_b &&
               (!PAGED || (c.g + 1) % cv.pg != 0)) {
        // two consecutive groups per stage, never across a page boundary
        nu = 2;
        np1 = unit_npos(cv, c, c.g + 1);
    }
    StageMeta m;
    m.b = c.b;
    m.vs = c.vs;
    m.npos = np0 | (np1 << 8);
    if (MODE == PREFIX) {
        // the stage's last segment ends the group, or the range
        const bool group_end = c.seg + nu == c.nseg, range_end = c.left == nu;
        m.flags = (c.seg == 0 ? STG_FIRST : 0) | (group_end || range_end ? STG_CLOSE : 0) |
                  (c.head ? STG_HEAD : 0) | (range_end && !group_end ? STG_HAND : 0);
    } else {
        m.flags = STG_FIRST | STG_CLOSE;
    }
    m.pos0 = FMT == DKV_FMT_DELTA ? c.g * cv.kf + c.seg * SEG : c.g * SEG;
    if (lane == 0) {
        if (KCfg<FMT, MODE>::NS > 1) *meta = m;
        issue_stage<FMT, MODE, PAGED>(cv, c, nhg, nu, np0 + np1, stage, bar, fault);
    }
    cursor_next<MODE>(c, cv, nvs, nhg);
    if (nu == 2) cursor_next<MODE>(c, cv, nvs, nhg);
    return m;
}


__device__ inline float q_elem(const void *Q, int dt, int64_t i) {
    if (dt == DKV_F32) return static_cast<const float *>(Q)[i];
    if (dt == DKV_F16) return __half2float(static_cast<const __half *>(Q)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(Q)[i]);
}

__device__ inline float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// Inclusive prefix over the 32 positions 4g + i (i = 0..3) of one head, held
// as v[i] by the 8 lanes g of one column (lane % 4).  Returns the total over
// the 32 positions (every lane).
__device__ inline float col_scan32(float (&v)[4], int lane) {
    v[1] += v[0];
    v[2] += v[1];
    v[3] += v[2];
    const float own = v[3];
    float inc = own;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    const float ex = inc - own;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] += ex;
    return __shfl_sync(0xffffffffu, inc, 28 + (lane & 3));
}

// Per unit (up to 32 positions), per thread of lane (g, t4):
//  K side, tile t: m16n8k16 with rows = positions (row g <-> 4g + 2t, row
//   g+8 <-> 4g + 2t + 1), k = channels, n = heads; the accumulator holds
//   x[t][r][e] for position 4g + 2t + r, head 2t4 + e, so each thread owns
//   the four consecutive positions 4g..4g+3 of two heads.
//  V side, tile t: m16n8k16 with rows = channels, k = positions
//   (k 2t4, 2t4+1 <-> 8t4 + 2t, +4; k 2t4+8, 2t4+9 <-> 8t4 + 2t + 1, +5),
//   n = heads; the weights reach that B layout through an 8x8 transpose
//   (movmatrix) of the K-side accumulator layout.

// K side of one unit: per-position dot products x[t][r][e] (position
// 4g + 2t + r, head 2tq + e).
// ZT: zero the scales of slots past the unit's end.  Needed where such a slot
// can read bytes that are not scale rows (kf < 32: the next record's nibbles,
// whose fp16 reading may be NaN); with kf = 32 and for Q4_0 a slot past the end
// reads a scale row of the cache (zeroed at init, else written by the encoder)
// or of an older stage, always finite, and the softmax mask alone handles it.
template <int FMT, int MODE, bool ZT, bool QHL>
__device__ inline void k_side(const uint8_t *st, const StageMap &sm, int npos, bool first_seg,
                              int gq, int tq, uint32_t m1024, uint32_t m64,
                              const uint32_t (&qb)[8][2], const uint32_t (&ql)[8][2],
                              const uint4 *qs, float (&x)[2][2][2]) {
    const bool kfrow = first_seg && gq == 0;   // this thread's row 0 of tile 0 is the keyframe
    // B fragments of q for k-steps 2j, 2j + 1: from registers, or (DKV_QSM)
    // from this lane's slots in shared memory
    auto qfrag = [&](int j, uint32_t &b0, uint32_t &b1, uint32_t &b2, uint32_t &b3) {
        if constexpr (DKV_QSM != 0 && !QHL) {
            const uint4 v = qs[j * 32 + 4 * gq + tq];
            b0 = v.x; b1 = v.y; b2 = v.z; b3 = v.w;
        } else {
            b0 = qb[2 * j][0]; b1 = qb[2 * j][1]; b2 = qb[2 * j + 1][0]; b3 = qb[2 * j + 1][1];
        }
    };
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int p0 = 4 * gq + 2 * t;             // positions p0, p0 + 1
        if (FMT == DKV_FMT_FP16) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const uint8_t *k0 = st + p0 * 256 + 64 * tq;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const uint4 u0 = *reinterpret_cast<const uint4 *>(k0 + 16 * q4);
                const uint4 u1 = *reinterpret_cast<const uint4 *>(k0 + 256 + 16 * q4);
                uint32_t b0, b1, b2, b3;
                qfrag(q4, b0, b1, b2, b3);
                mma16816(acc, u0.x, u1.x, u0.y, u1.y, b0, b1);
                mma16816(acc, u0.z, u1.z, u0.w, u1.w, b2, b3);
                if (QHL) {
                    mma16816(acc, u0.x, u1.x, u0.y, u1.y, ql[2 * q4][0], ql[2 * q4][1]);
                    mma16816(acc, u0.z, u1.z, u0.w, u1.w, ql[2 * q4 + 1][0], ql[2 * q4 + 1][1]);
                }
            }
            x[t][0][0] = acc[0]; x[t][0][1] = acc[1];
            x[t][1][0] = acc[2]; x[t][1][1] = acc[3];
        } else {
            const uint4 w0 = *reinterpret_cast<const uint4 *>(st + sm.kn0 + p0 * NIB_BYTES + 16 * tq);
            const uint4 w1 = *reinterpret_cast<const uint4 *>(st + sm.kn0 + (p0 + 1) * NIB_BYTES + 16 * tq);
            uint32_t a[8][4];
            {
                const uint32_t ww0[4] = {w0.x, w0.y, w0.z, w0.w};
                const uint32_t ww1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    dq_word(ww0[j], m1024, m64, a[2 * j][0], a[2 * j][2], a[2 * j + 1][0],
                            a[2 * j + 1][2]);
                    dq_word(ww1[j], m1024, m64, a[2 * j][1], a[2 * j][3], a[2 * j + 1][1],
                            a[2 * j + 1][3]);
                }
            }
            if (FMT == DKV_FMT_DELTA && t == 0 && first_seg && kfrow) {
                // position 0 is the keyframe: its fp16 values fill rows g = 0
                // (loaded by those lanes only, straight into the A fragment)
                const uint8_t *kp = st + sm.kf0 + 64 * tq;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(kp + 16 * q4);
                    a[2 * q4][0] = v.x;
                    a[2 * q4][2] = v.y;
                    a[2 * q4 + 1][0] = v.z;
                    a[2 * q4 + 1][2] = v.w;
                }
            }
            float acc[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                uint32_t b0, b1, b2, b3;
                qfrag(j, b0, b1, b2, b3);
                mma16816(acc[j], a[2 * j][0], a[2 * j][1], a[2 * j][2], a[2 * j][3], b0, b1);
                mma16816(acc[j], a[2 * j + 1][0], a[2 * j + 1][1], a[2 * j + 1][2],
                         a[2 * j + 1][3], b2, b3);
                if (QHL) {
                    mma16816(acc[j], a[2 * j][0], a[2 * j][1], a[2 * j][2], a[2 * j][3],
                             ql[2 * j][0], ql[2 * j][1]);
                    mma16816(acc[j], a[2 * j + 1][0], a[2 * j + 1][1], a[2 * j + 1][2],
                             a[2 * j + 1][3], ql[2 * j + 1][0], ql[2 * j + 1][1]);
                }
            }
            // K scales of positions p0, p0+1 (blocks 0..3; the V scales
            // follow in the same 16-byte row and are read by the V side)
            uint2 s0 = *reinterpret_cast<const uint2 *>(st + sm.sc0 + p0 * SC_BYTES);
            uint2 s1 = *reinterpret_cast<const uint2 *>(st + sm.sc0 + (p0 + 1) * SC_BYTES);
            if (FMT == DKV_FMT_DELTA && t == 0 && kfrow) s0.x = s0.y = 0x3C003C00u;  // keyframe: unit
            if (ZT) {
                if (p0 >= npos) s0 = make_uint2(0u, 0u);
                if (p0 + 1 >= npos) s1 = make_uint2(0u, 0u);
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float x0 = acc[0][e] * h_lo(s0.x);
                x0 = fmaf(acc[1][e], h_hi(s0.x), x0);
                x0 = fmaf(acc[2][e], h_lo(s0.y), x0);
                x[t][0][e] = fmaf(acc[3][e], h_hi(s0.y), x0);
                float x1 = acc[0][2 + e] * h_lo(s1.x);
                x1 = fmaf(acc[1][2 + e], h_hi(s1.x), x1);
                x1 = fmaf(acc[2][2 + e], h_lo(s1.y), x1);
                x[t][1][e] = fmaf(acc[3][2 + e], h_hi(s1.y), x1);
            }
        }
    }
}

// V side of one unit: o += sum over positions of dequantised V rows times the
// weights w[t][r][e] (position 4g + 2t + r, head 2tq + e) and their V scales.
// The V scales are read here rather than kept from the K side (registers).
template <int FMT, int MODE, bool ZT, bool RC>
__device__ inline void v_side(const uint8_t *st, const StageMap &sm, int npos, bool first_seg,
                              int gq, int tq, uint32_t m1024, uint32_t m64,
                              const float (&w)[2][2][2], float (&o)[8][4], float (&racc)[8][4],
                              uint32_t (&vkf_keep)[8]) {
    uint32_t vkf[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (FMT == DKV_FMT_DELTA && first_seg) {
        const uint4 v0 = *reinterpret_cast<const uint4 *>(st + sm.vk0 + 32 * gq);
        const uint4 v1 = *reinterpret_cast<const uint4 *>(st + sm.vk0 + 32 * gq + 16);
        vkf[0] = v0.x; vkf[1] = v0.y; vkf[2] = v0.z; vkf[3] = v0.w;
        vkf[4] = v1.x; vkf[5] = v1.y; vkf[6] = v1.z; vkf[7] = v1.w;
        if (MODE == PREFIX) {
#pragma unroll
            for (int i = 0; i < 8; ++i) vkf_keep[i] = vkf[i];
        }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        if (FMT == DKV_FMT_FP16) {
            // one token per row: one fp16 weight, as flash-decoding does
            uint32_t bp[2];
            bp[0] = movm_t(pack_h2(w[t][0][0], w[t][0][1]));
            bp[1] = movm_t(pack_h2(w[t][1][0], w[t][1][1]));
            // V values of positions 8tq + 2t + {0, 1, 4, 5}, chunk g
            const uint8_t *vb = st + 8192 + (8 * tq + 2 * t) * 256 + 32 * gq;
            uint32_t wv[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int dp = (i & 1) + 4 * (i >> 1);
                const uint4 lo4 = *reinterpret_cast<const uint4 *>(vb + dp * 256);
                const uint4 hi4 = *reinterpret_cast<const uint4 *>(vb + dp * 256 + 16);
                wv[i][0] = lo4.x; wv[i][1] = lo4.y; wv[i][2] = lo4.z; wv[i][3] = lo4.w;
                wv[i][4] = hi4.x; wv[i][5] = hi4.y; wv[i][6] = hi4.z; wv[i][7] = hi4.w;
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const uint32_t a0 = prmt(wv[0][mt], wv[2][mt], 0x5410u);
                const uint32_t a1 = prmt(wv[0][mt], wv[2][mt], 0x7632u);
                const uint32_t a2 = prmt(wv[1][mt], wv[3][mt], 0x5410u);
                const uint32_t a3 = prmt(wv[1][mt], wv[3][mt], 0x7632u);
                mma16816(o[mt], a0, a1, a2, a3, bp[0], bp[1]);
            }
            continue;
        }
        // V scales of positions 4g + 2t + r (the weights' positions).  On the
        // keyframe row: 1 for whole groups (v_f rides the MMA, below), 0 for
        // segments (kf > 32: v_f is added when the group closes).  With ZT, 0
        // on slots past the unit's end.
        uint32_t dvw[2][2];
        {
            const int p0 = 4 * gq + 2 * t;
            uint2 s0 = *reinterpret_cast<const uint2 *>(st + sm.sc0 + p0 * SC_BYTES + 8);
            uint2 s1 = *reinterpret_cast<const uint2 *>(st + sm.sc0 + (p0 + 1) * SC_BYTES + 8);
            if (FMT == DKV_FMT_DELTA && t == 0 && first_seg && gq == 0)
                s0 = MODE == PREFIX ? make_uint2(0u, 0u) : make_uint2(0x3C003C00u, 0x3C003C00u);
            if (ZT) {
                if (p0 >= npos) s0 = make_uint2(0u, 0u);
                if (p0 + 1 >= npos) s1 = make_uint2(0u, 0u);
            }
            dvw[0][0] = s0.x; dvw[0][1] = s0.y;
            dvw[1][0] = s1.x; dvw[1][1] = s1.y;
        }
        // V nibbles of positions 8tq + 2t + {0, 1, 4, 5}, chunk g
        const uint8_t *vb = st + sm.vn0 + (8 * tq + 2 * t) * NIB_BYTES + 8 * gq;
        const uint2 wP0 = *reinterpret_cast<const uint2 *>(vb);
        const uint2 wP1 = *reinterpret_cast<const uint2 *>(vb + NIB_BYTES);
        const uint2 wP2 = *reinterpret_cast<const uint2 *>(vb + 4 * NIB_BYTES);
        const uint2 wP3 = *reinterpret_cast<const uint2 *>(vb + 5 * NIB_BYTES);
        // A fragment of m-tile mt: exact code - 8 of channels 16mt + g (rows g)
        // and 16mt + g + 8 (rows g + 8), k pairs (pos 8tq+2t, +4) | (+1, +5)
        auto codes = [&](int mt, uint32_t &a0, uint32_t &a1, uint32_t &a2, uint32_t &a3) {
            const int i = mt & 3;
            const uint32_t sel = (uint32_t)(i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12));
            const uint32_t m01 = prmt(mt < 4 ? wP0.x : wP0.y, mt < 4 ? wP2.x : wP2.y, sel);
            const uint32_t m23 = prmt(mt < 4 ? wP1.x : wP1.y, mt < 4 ? wP3.x : wP3.y, sel);
            dq_pair(m01, m1024, m64, a0, a1);
            dq_pair(m23, m1024, m64, a2, a3);
        };
        if (MODE != PREFIX) {
            // B fragments (k = positions, n = head g) of block j: the weight of
            // each row times block j's V scale, then the 8x8 transpose into the
            // B layout.  Delta format: the weights are suffix sums S_s, and the
            // terms delta^_s * S_s cancel to the much smaller output whenever
            // consecutive tokens differ a lot (jumps, unrelated tokens), so one
            // fp16 value of S_s * d_s (relative error 2^-11) can give outputs
            // off by 1 %.  There every B value is an fp16 pair hi + lo:
            //   hi = fp16(fp16(S) * d);  lo = fp16(fp16(S - fp16(S)) * d +
            //   (fp16(S) * d - hi)), the bracket exact (one fused multiply-add
            //   returns the rounding error of a product exactly),
            // with the second MMA against the same A fragment, for a relative
            // error near 2^-21.  The comparators (one token per row) keep one
            // fp16 weight, as flash-decoding does.
            constexpr bool HL = FMT == DKV_FMT_DELTA;
            const uint32_t wp0 = pack_h2(w[t][0][0], w[t][0][1]);
            const uint32_t wp1 = pack_h2(w[t][1][0], w[t][1][1]);
            uint32_t wl0 = 0, wl1 = 0;
            if (HL) {
                wl0 = pack_h2(w[t][0][0] - h_lo(wp0), w[t][0][1] - h_hi(wp0));
                wl1 = pack_h2(w[t][1][0] - h_lo(wp1), w[t][1][1] - h_hi(wp1));
            }
            auto make_b = [&](int j, uint32_t (&b)[2], uint32_t (&bl)[2]) {
                const uint32_t u0 = dvw[0][j >> 1], u1 = dvw[1][j >> 1];
                const __half2 d0 = (j & 1) ? __high2half2(u32_as_h2(u0)) : __low2half2(u32_as_h2(u0));
                const __half2 d1 = (j & 1) ? __high2half2(u32_as_h2(u1)) : __low2half2(u32_as_h2(u1));
                const __half2 h0 = __hmul2(u32_as_h2(wp0), d0);
                const __half2 h1 = __hmul2(u32_as_h2(wp1), d1);
                b[0] = movm_t(h2_as_u32(h0));
                b[1] = movm_t(h2_as_u32(h1));
                if (HL) {
                    const __half2 l0 = __hfma2(u32_as_h2(wl0), d0,
                                               __hfma2(u32_as_h2(wp0), d0, __hneg2(h0)));
                    const __half2 l1 = __hfma2(u32_as_h2(wl1), d1,
                                               __hfma2(u32_as_h2(wp1), d1, __hneg2(h1)));
                    bl[0] = movm_t(h2_as_u32(l0));
                    bl[1] = movm_t(h2_as_u32(l1));
                }
            };
            // Delta format: slot 0 of tile 0 is the keyframe position, which has
            // no delta row; its A entries (the low halves of a0 / a1 on the
            // lanes with tq = 0) take v_f itself, and its scale is 1, so the
            // MMA adds v_f times the group's total weight (S of position 0).
            const bool kf_slot = FMT == DKV_FMT_DELTA && t == 0 && first_seg && tq == 0;
            uint32_t bp[2], bq[2] = {0u, 0u};
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t a0, a1, a2, a3;
                codes(mt, a0, a1, a2, a3);
                if (kf_slot) {
                    a0 = prmt(a0, vkf[mt], 0x3254u);   // channel 16mt + g
                    a1 = prmt(a1, vkf[mt], 0x3276u);   // channel 16mt + g + 8
                }
                if ((mt & 1) == 0) make_b(mt >> 1, bp, bq);
                mma16816(o[mt], a0, a1, a2, a3, bp[0], bp[1]);
                if (HL) mma16816(o[mt], a0, a1, a2, a3, bq[0], bq[1]);
            }
        } else {
            // PREFIX (kf > 32): the prefix weights -E_s aggregate up to kf
            // positions; every B value is an fp16 hi + lo pair, made as for
            // whole groups (above), and a third MMA against the scales alone
            // (exact fp16 values) sums the group's dequantised deltas R_g.
            const uint32_t wp0 = pack_h2(w[t][0][0], w[t][0][1]);
            const uint32_t wp1 = pack_h2(w[t][1][0], w[t][1][1]);
            const uint32_t wl0 = pack_h2(w[t][0][0] - h_lo(wp0), w[t][0][1] - h_hi(wp0));
            const uint32_t wl1 = pack_h2(w[t][1][0] - h_lo(wp1), w[t][1][1] - h_hi(wp1));
            auto make_b = [&](int j, uint32_t (&b)[2], uint32_t (&bl)[2], uint32_t (&rr)[2]) {
                const uint32_t u0 = dvw[0][j >> 1], u1 = dvw[1][j >> 1];
                const __half2 d0 = (j & 1) ? __high2half2(u32_as_h2(u0)) : __low2half2(u32_as_h2(u0));
                const __half2 d1 = (j & 1) ? __high2half2(u32_as_h2(u1)) : __low2half2(u32_as_h2(u1));
                const __half2 h0 = __hmul2(u32_as_h2(wp0), d0);
                const __half2 h1 = __hmul2(u32_as_h2(wp1), d1);
                const __half2 l0 = __hfma2(u32_as_h2(wl0), d0,
                                           __hfma2(u32_as_h2(wp0), d0, __hneg2(h0)));
                const __half2 l1 = __hfma2(u32_as_h2(wl1), d1,
                                           __hfma2(u32_as_h2(wp1), d1, __hneg2(h1)));
                b[0] = movm_t(h2_as_u32(h0));
                b[1] = movm_t(h2_as_u32(h1));
                bl[0] = movm_t(h2_as_u32(l0));
                bl[1] = movm_t(h2_as_u32(l1));
                rr[0] = movm_t(h2_as_u32(d0));
                rr[1] = movm_t(h2_as_u32(d1));
            };
            uint32_t bp[2], bl[2], rr[2];
            if constexpr (RC) {
                // columns 4-7 (threads tq >= 2 before the transpose): the V
                // scale itself in the hi operand and 0 in the lo one, so those
                // accumulator columns sum the dequantised deltas
                const bool rcol = tq >= 2;
                auto make_b_rc = [&](int j, uint32_t (&b)[2], uint32_t (&bl)[2]) {
                    const uint32_t u0 = dvw[0][j >> 1], u1 = dvw[1][j >> 1];
                    const __half2 d0 = (j & 1) ? __high2half2(u32_as_h2(u0)) : __low2half2(u32_as_h2(u0));
                    const __half2 d1 = (j & 1) ? __high2half2(u32_as_h2(u1)) : __low2half2(u32_as_h2(u1));
                    const __half2 h0 = __hmul2(u32_as_h2(wp0), d0);
                    const __half2 h1 = __hmul2(u32_as_h2(wp1), d1);
                    const __half2 l0 = __hfma2(u32_as_h2(wl0), d0,
                                               __hfma2(u32_as_h2(wp0), d0, __hneg2(h0)));
                    const __half2 l1 = __hfma2(u32_as_h2(wl1), d1,
                                               __hfma2(u32_as_h2(wp1), d1, __hneg2(h1)));
                    b[0] = movm_t(h2_as_u32(rcol ? d0 : h0));
                    b[1] = movm_t(h2_as_u32(rcol ? d1 : h1));
                    bl[0] = movm_t(rcol ? 0u : h2_as_u32(l0));
                    bl[1] = movm_t(rcol ? 0u : h2_as_u32(l1));
                };
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    uint32_t a0, a1, a2, a3;
                    codes(mt, a0, a1, a2, a3);
                    if ((mt & 1) == 0) make_b_rc(mt >> 1, bp, bl);
                    mma16816(o[mt], a0, a1, a2, a3, bp[0], bp[1]);
                    mma16816(o[mt], a0, a1, a2, a3, bl[0], bl[1]);
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    uint32_t a0, a1, a2, a3;
                    codes(mt, a0, a1, a2, a3);
                    if ((mt & 1) == 0) make_b(mt >> 1, bp, bl, rr);
                    mma16816(o[mt], a0, a1, a2, a3, bp[0], bp[1]);
                    mma16816(o[mt], a0, a1, a2, a3, bl[0], bl[1]);
                    mma16816(racc[mt], a0, a1, a2, a3, rr[0], rr[1]);   // R += (code - 8) d
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Fused append (delta format).  The n new tokens of sequence (b, kv head) are
// quantised inside the split kernel by the warps whose unit ranges hold the
// groups they land in, before those warps copy any record: each such warp runs
// the closed loop of the method (page "...Delta-KV", section "핵심 아이디어":
// keyframe at p mod kf == 0, else a Q4_0 delta from the reconstruction of
// p - 1) over the new tokens from the stored reconstruction, and stores the
// fields of the positions in its own groups.  Every quantiser step is the
// encoder's, in the same order, so the stored fields are the ones the
// separate append would write.  A warp of another head group of the same kv
// head (multi-query, more than 8 virtual heads) stores the same bytes again;
// each warp reads the records only after its own stores.  The reconstruction
// after the last token goes to the other state slot, which the merge makes
// current.
// ---------------------------------------------------------------------------
// Input element c of row `row` of an n-token K_new / V_new array.
__device__ inline float load_new(const void *src, int dtype, int64_t row, int c) {
    const int64_t i = row * D + c;
    if (dtype == DKV_F16) return __half2float(__ldg(static_cast<const __half *>(src) + i));
    if (dtype == DKV_BF16)
        return __bfloat162float(__ldg(static_cast<const __nv_bfloat16 *>(src) + i));
    return __ldg(static_cast<const float *>(src) + i);
}

template <bool PAGED>
__device__ __noinline__ void append_tokens(const SplitArgs &A, int b, int kvh, int L0, int p_lo,
                                           int p_hi, bool write_state) {
    const CacheView &cv = A.cv;
    const int lane = threadIdx.x & 31, kf = cv.kf, n = cv.len_add;
    const int64_t sb = ((int64_t)b * cv.Hkv + kvh) * 2 * D;          // (b, kvh) in a slot
    const int64_t slot = (int64_t)cv.B * cv.Hkv * 2 * D;
    const int64_t row0 = ((int64_t)b * cv.Hkv + kvh) * n;
    // checked build: the sequence's state in both slots and its n input rows
    if (DKV_CHECKED) {
        const int ies = A.kv_dtype == DKV_F32 ? 4 : 2;
        const int64_t in_bytes = (int64_t)cv.B * cv.Hkv * n * D * ies;
        if (!state_ok(cv, cv.state + sb, 2 * D) || !state_ok(cv, cv.state + slot + sb, 2 * D) ||
            !range_ok(cv.header, static_cast<const uint8_t *>(A.Kn) + row0 * D * ies,
                      (int64_t)n * D * ies, A.Kn, in_bytes) ||
            !range_ok(cv.header, static_cast<const uint8_t *>(A.Vn) + row0 * D * ies,
                      (int64_t)n * D * ies, A.Vn, in_bytes))
            return;
    }
    // one round trip: the slot word, both state slots and the first token
    const int parity = cv.header[2] & 1;
    const bool cont = (L0 % kf) != 0;            // the first token continues a group
    float s0[2][4], s1[2][4], x[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t e = sb + t * D + 32 * j + lane;
            s0[t][j] = cont ? __ldg(cv.state + e) : 0.f;
            s1[t][j] = cont ? __ldg(cv.state + slot + e) : 0.f;
            x[t][j] = load_new(t ? A.Vn : A.Kn, A.kv_dtype, row0, 32 * j + lane);
        }
    float xh[2][4];                     // reconstruction of channels 32 j + lane, K and V
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) xh[t][j] = parity ? s1[t][j] : s0[t][j];
    float *st_new = cv.state + (parity ^ 1) * slot + sb;
    // this lane's nibble word: K word `lane` (lanes 0-15) or V word lane - 16
    const int wt = lane >> 4, ww = lane & 15;
#pragma unroll 1
    for (int i = 0; i < n; ++i) {
        const int p = L0 + i, g = p / kf, di = p - g * kf;   // di 0: keyframe; else delta di - 1
        if (p >= p_hi) break;
        uint8_t *rec = p >= p_lo ? rec_ptr<PAGED>(cv, b, kvh, g) : nullptr;
        if (rec && !rec_ok(cv, rec, cv.rec_bytes)) rec = nullptr;   // checked build
        if (di == 0) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half h = __float2half_rn(x[t][j]);
                    xh[t][j] = __half2float(h);
                    const int ch = 32 * j + lane;
                    if (rec)
                        reinterpret_cast<__half *>(rec + t * 256)[t == 0 ? k_half_idx(ch)
                                                                         : v_half_idx(ch)] = h;
                }
        } else {
            // the eight blocks (K and V, 4 each) are independent chains
            uint32_t codes = 0;         // code of channel 32 j + lane of tensor t at bit 16 t + 4 j
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
                xh[t][j] = __fadd_rn(xh[t][j], __fmul_rn((float)(cd[i] - 8), __half2float(h16[i])));
            }
            if (rec) {
                // gather the 8 codes of this lane's word from the lanes holding them
                uint32_t word = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int ch = nib_channel(wt, ww, k);
                    const uint32_t v = __shfl_sync(0xffffffffu, codes, ch & 31);
                    word |= ((v >> (16 * wt + 4 * (ch >> 5))) & 15u) << (4 * k);
                }
                uint8_t *nib = rec + KF_BYTES + (int64_t)(kf - 1) * SC_BYTES +
                               ((int64_t)wt * (kf - 1) + (di - 1)) * NIB_BYTES;
                reinterpret_cast<uint32_t *>(nib)[ww] = word;
                if (lane < 2) {
                    uint2 v;
                    v.x = (uint32_t)__half_as_ushort(d16[lane][0]) |
                          ((uint32_t)__half_as_ushort(d16[lane][1]) << 16);
                    v.y = (uint32_t)__half_as_ushort(d16[lane][2]) |
                          ((uint32_t)__half_as_ushort(d16[lane][3]) << 16);
                    *reinterpret_cast<uint2 *>(rec + KF_BYTES + (int64_t)(di - 1) * SC_BYTES +
                                               lane * 8) = v;
                }
            }
        }
        if (i + 1 < n) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    x[t][j] = load_new(t ? A.Vn : A.Kn, A.kv_dtype, row0 + i + 1, 32 * j + lane);
        }
    }
    if (write_state) {
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) st_new[t * D + 32 * j + lane] = xh[t][j];
    }
}

// The new tokens that land in units [lo, hi) of a warp's range (offsets from
// the range's first unit, which is unit u0 of sequence vs of batch entry b, a
// sequence of ub units): walk the sequences those units belong to and
// quantise, for each, the new tokens from the first one on, storing those at
// the positions of the units held there.  The owner of a sequence's last unit
// (head group 0) writes the state.  Returns whether this warp stored anything.
template <bool PAGED>
__device__ __noinline__ bool append_range(const SplitArgs &A, int nvs, int b, int vs, int u0,
                                          int ub, int64_t lo, int64_t hi) {
    const CacheView &cv = A.cv;
    bool wrote = false;
    int64_t off = 0;                    // offset of unit u0 of (b, vs) in the range
#pragma unroll 1
    while (off < hi) {
        const int64_t here = ub - u0;   // units of this sequence from u0 on
        if (off + here > lo) {
            const int ua = u0 + (int)max((int64_t)0, lo - off);
            const int ue = u0 + (int)(min(hi, off + here) - off);       // exclusive
            int L;
            if (takes_append(cv, b, L)) {
                const int p_lo = max((int)unit_pos(cv.fmt, cv.kf, ua), L);
                const int p_hi = min((int)unit_pos(cv.fmt, cv.kf, ue), L + cv.len_add);
                if (p_lo < p_hi) {
                    append_tokens<PAGED>(A, b, A.NHG == 1 ? vs : vs / A.NHG, L, p_lo, p_hi,
                                         ue == ub && vs % A.NHG == 0);
                    wrote = true;
                }
            }
        }
        off += here;
        if (off >= hi) break;
        u0 = 0;
        if (++vs == nvs) {
            vs = 0;
            do {
                if (++b >= cv.B) return wrote;
                ub = units_of(cv.fmt, cv.kf, clamp_len(cv, b));
            } while (ub == 0);
        }
    }
    return wrote;
}

// MQ: several causal queries per sequence (virtual heads with their own
// position limits); the one-query instance keeps the plain tail mask.  APP:
// the fused append (the kernel parameters stay in the constant bank while the
// append functions take their address).  QHL: fp32 queries as an fp16 hi + lo
// pair (two MMAs per K-side step; the extra registers cost a CTA per SM).
// RC (kf > 32, at most 4 heads per head group): the group's sum of dequantised
// V deltas R_g accumulates in the output accumulators' columns 4-7, which no
// head uses (their B operand is the V scale), instead of 32 registers of its own.
template <int FMT, int MODE, bool ZT, bool PAGED, bool MQ, bool APP, bool QHL, bool RC = false>
__global__ void __launch_bounds__(WARPS * 32, (QHL ? 2 : KCfg<FMT, MODE>::MINB))
    split_kernel(const __grid_constant__ SplitArgs A) {
    using Cfg = KCfg<FMT, MODE>;
    constexpr int NS = Cfg::NS, STAGE = Cfg::STAGE, NU = Cfg::NU;
    using Map = SmemMap<FMT, MODE>;
    extern __shared__ __align__(1024) uint8_t smem[];

    const CacheView &cv = A.cv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;          // quad row / column of the fragments
    const int nvs = cv.Hkv * A.NHG;                    // sequences per batch entry
    uint64_t *mybar = reinterpret_cast<uint64_t *>(smem + Map::BAR_OFF) + warp * NS;
    StageMeta *mymeta = reinterpret_cast<StageMeta *>(smem + Map::META_OFF) + warp * NS;
    uint8_t *mystages = smem + Map::STAGE_OFF + warp * NS * STAGE;
    uint4 *myq = reinterpret_cast<uint4 *>(smem + Map::Q_OFF) + warp * 128;   // DKV_QSM
    const uint32_t m1024 = magic_1024x2(), m64 = magic_64x2();

    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(mybar + s, 1);
        fence_mbar_init();
    }
    // zero the stages once so slots no copy has filled hold finite values
    for (int i = lane; i < NS * STAGE / 16; i += 32)
        reinterpret_cast<uint4 *>(mystages)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    __syncwarp();
    pdl_trigger();
    pdl_wait();           // every global access below follows the previous kernel

    const int64_t NW = (int64_t)gridDim.x * WARPS;
    const int64_t gw = (int64_t)blockIdx.x * WARPS + warp;
    int bdummy;
    int64_t base_dummy;
    const int64_t total = locate(cv, nvs, -1, bdummy, base_dummy);
    if constexpr (APP) {
        if (gw == 0) {
            // the lengths this call decodes, for the merge (which publishes
            // the new ones); an entry that takes no tokens keeps its
            // reconstruction: carry it into the slot the merge makes current
            int32_t *lenv = merge_lengths(A.ws, NW, cv.B * nvs);
            if (range_ok(cv.header, lenv, (int64_t)cv.B * 4, A.ws, A.ws_floats * 4))
                for (int b = lane; b < cv.B; b += 32) lenv[b] = clamp_len(cv, b);
            const int parity = cv.header[2] & 1;
            const int64_t per_b = (int64_t)cv.Hkv * 2 * D;
            for (int b = 0; b < cv.B; ++b) {
                int l;
                if (takes_append(cv, b, l)) continue;
                if (lane == 0)
                    set_status(cv.header, (l < 0 || l > cv.cap) ? DKV_DEV_BAD_SEQLEN
                                                                : DKV_DEV_CAPACITY);
                const float *so = cv.state + ((int64_t)parity * cv.B + b) * per_b;
                float *sn = cv.state + ((int64_t)(parity ^ 1) * cv.B + b) * per_b;
                for (int64_t k = lane; k < per_b; k += 32) sn[k] = so[k];
            }
        }
    } else {
        if (gw == 0 && lane == 0) {
            for (int b = 0; b < cv.B; ++b) {
                const int l = cv.seqlen[b];
                if (l < 0 || l > cv.cap) set_status(cv.header, DKV_DEV_BAD_SEQLEN);
            }
        }
    }
    if (MODE == PREFIX && gw == 0 && lane == 0 && range_ok(cv.header, A.hands, 4, A.ws, A.ws_floats * 4))
        A.hands[0] = A.scale_log2;   // for the merge
    if (total == 0) return;
    const int64_t r0 = range_start(gw, NW, total), r1 = range_start(gw + 1, NW, total);
    if (r0 >= r1) return;

    Cursor ic;
    cursor_seek<MODE>(ic, cv, nvs, A.NHG, r0, r1 - r0);
    // fused append: tokens landing in the units the first NS stages can hold
    // are stored before those copies are issued; the rest after, while the
    // first copies are in flight (each warp copies a record only after its
    // own stores and a proxy fence)
    const int ab = ic.b, avs = ic.vs, aub = ic.units_b;
    const int ag = MODE == PREFIX ? ic.g * seg_per_group(cv.kf) + ic.seg : ic.g;   // unit
    constexpr int64_t PRE = (int64_t)NS * NU;
    if constexpr (APP) {
        if (append_range<PAGED>(A, nvs, ab, avs, ag, aub, 0, min(PRE, r1 - r0))) {
            fence_proxy_async_global();
            __syncwarp();
        }
    }

    // prologue: fill the ring
    uint32_t phase = 0;                 // bit s = parity to wait for on stage s
    int issued = 0, consumed = 0;
    StageMeta pend{};                   // NS == 1: the issued stage's descriptor
#pragma unroll 1
    for (int s = 0; s < NS; ++s) {
        if (ic.valid()) {
            pend = next_stage<FMT, MODE, PAGED>(cv, ic, nvs, A.NHG, mystages + s * STAGE, mybar + s,
                                         mymeta + s, lane, A.fault);
            ++issued;
        }
    }
    if constexpr (APP) {
        if (r1 - r0 > PRE &&
            append_range<PAGED>(A, nvs, ab, avs, ag, aub, PRE, r1 - r0)) {
            fence_proxy_async_global();
            __syncwarp();
        }
    }

    bool dead = false;
    int stage_i = 0;

    // per-sequence state (heads 2*tq + e of the current head group)
    int cur_b = -1, cur_vs = -1;
    uint32_t qb[8][2];                  // B fragments of q (column = head gq)
    uint32_t ql[8][2];                  // QHL: the fp16 remainders q - qb
    int lp[2] = {0, 0};                 // positions heads 2tq + e may see (causal queries)
    float m_run[2] = {-1e30f, -1e30f}, l_run[2] = {0.f, 0.f};
    float o[8][4];
    float racc[8][4];                   // PREFIX: sum of dequantised deltas of the group
    float dot_carry[2] = {0.f, 0.f}, e_carry[2] = {0.f, 0.f};
    uint32_t vkf_keep[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { o[i][j] = 0.f; racc[i][j] = 0.f; }
#pragma unroll
    for (int i = 0; i < 8; ++i) vkf_keep[i] = 0;

    auto write_record = [&](float *rec) {
        // the partial record (m, l, o) of heads 2tq, 2tq + 1 (l summed over
        // the warp here)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float l = l_run[e];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            l_run[e] = l;
        }
        // checked build: the record inside the workspace (uniform over the warp)
        if (!range_ok(cv.header, rec, PARTIAL_FLOATS * 4, A.ws, A.ws_floats * 4)) return;
        if (gq == 0) {
            rec[2 * tq] = m_run[0];
            rec[2 * tq + 1] = m_run[1];
            rec[8 + 2 * tq] = l_run[0];
            rec[8 + 2 * tq + 1] = l_run[1];
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
    // the partial record of the current sequence
    auto flush = [&]() {
        write_record(A.ws + (gw + (int64_t)cur_b * nvs + cur_vs) * PARTIAL_FLOATS);
    };

#pragma unroll 1
    while (consumed < issued) {
        // ---- wait for the stage -------------------------------------------
        const uint8_t *st = mystages + stage_i * STAGE;
        if (!mbar_wait_bounded(mybar + stage_i, (phase >> stage_i) & 1)) {
            dead = true;
            if (lane == 0) set_status(cv.header, DKV_DEV_TIMEOUT);
        }
        // a warp that gave up leaves the loop with this stage's copies (and any
        // later ones) in flight; they are waited for below
        dead = __any_sync(0xffffffffu, dead);
        if (dead) break;
        phase ^= 1u << stage_i;
        const StageMeta meta = NS == 1 ? pend : mymeta[stage_i];

        // ---- sequence change: flush, load q --------------------------------
        if (meta.b != cur_b || meta.vs != cur_vs) {
            if (cur_b >= 0) flush();
            cur_b = meta.b; cur_vs = meta.vs;
            // virtual heads of a kv head: query t of the sequence, head h of the
            // GQA group -> v = t * G + h, 8 per head group; query t sees the
            // positions before len - (nq - 1 - t)
            const int kvh = meta.vs / A.NHG, hg = meta.vs % A.NHG;
            const int Gv = A.nq * A.G;
            const int vq = hg * 8 + gq;                  // virtual head of this thread's q column
            const bool qok = vq < Gv;
            const int qt = qok ? vq / A.G : 0, hl = qok ? vq % A.G : 0;
            const int len_b = clamp_len(cv, meta.b);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int ve = hg * 8 + 2 * tq + e;
                lp[e] = ve < Gv ? len_b - (A.nq - 1 - ve / A.G) : 0;   // absent head: none
            }
            const int64_t qrow =
                (((int64_t)meta.b * A.nq + qt) * A.Hq + (int64_t)kvh * A.G + hl) * D;
            // checked build: the q row inside Q ([B][nq][Hq][D] of q_dtype)
            const int qes = A.q_dtype == DKV_F32 ? 4 : 2;
            const bool q_in = !qok || range_ok(cv.header, static_cast<const uint8_t *>(A.Q) + qrow * qes,
                                               (int64_t)D * qes, A.Q,
                                               (int64_t)cv.B * A.nq * A.Hq * D * qes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c = 16 * kk + 2 * tq;
                float q0 = 0.f, q1 = 0.f, q8 = 0.f, q9 = 0.f;
                if (qok && q_in) {
                    q0 = q_elem(A.Q, A.q_dtype, qrow + c);
                    q1 = q_elem(A.Q, A.q_dtype, qrow + c + 1);
                    q8 = q_elem(A.Q, A.q_dtype, qrow + c + 8);
                    q9 = q_elem(A.Q, A.q_dtype, qrow + c + 9);
                }
                qb[kk][0] = pack_h2(q0, q1);
                qb[kk][1] = pack_h2(q8, q9);
                if (DKV_QSM != 0 && !QHL && (kk & 1)) {
                    // this lane's own slots: no other lane reads them
                    myq[(kk >> 1) * 32 + lane] =
                        make_uint4(qb[kk - 1][0], qb[kk - 1][1], qb[kk][0], qb[kk][1]);
                }
                if (QHL) {
                    // fp32 queries: q = hi + lo, both fp16, so q . k keeps
                    // about 22 bits (bf16 and fp16 queries are exact in hi)
                    ql[kk][0] = pack_h2(q0 - h_lo(qb[kk][0]), q1 - h_hi(qb[kk][0]));
                    ql[kk][1] = pack_h2(q8 - h_lo(qb[kk][1]), q9 - h_hi(qb[kk][1]));
                }
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                m_run[e] = -1e30f; l_run[e] = 0.f; dot_carry[e] = 0.f; e_carry[e] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) { o[i][j] = 0.f; racc[i][j] = 0.f; }
        }

        {
            int npos[NU];
#pragma unroll
            for (int u = 0; u < NU; ++u) npos[u] = (meta.npos >> (8 * u)) & 0xff;
            // kf <= 32: every unit is a whole group, so it starts with its keyframe
            const bool first_seg = (FMT == DKV_FMT_DELTA) && (MODE == SUFFIX || (meta.flags & 1));
            const bool last_seg = MODE != PREFIX || (meta.flags & 2) != 0;

            // ================= K side ======================================
            float x[NU][2][2][2];
            // Both units go through the same straight-line code; a unit the stage
            // does not hold has npos 0, so all its slots are masked and its scales
            // zeroed (its shared-memory bytes are an older stage's, always finite).
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                const StageMap sm = stage_map<FMT, MODE>(cv.kf, cv.rec_bytes, u);
                // kf > 32: only a stage's first segment can hold a keyframe
                k_side<FMT, MODE, ZT, QHL>(st, sm, npos[u], first_seg && (MODE != PREFIX || u == 0),
                                           gq, tq, m1024, m64, qb, ql, myq, x[u]);
            }

            // ================= scores, online softmax =======================
            // valid slots of this thread per head: positions 4g + i with i < lim[u][e]
            // (the unit's end, and for causal queries the head's own limit)
            int lim[NU][2];
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                if (MQ) {
                    const int us = meta.pos0 + u * (MODE == SUFFIX ? cv.kf : SEG);
#pragma unroll
                    for (int e = 0; e < 2; ++e) lim[u][e] = min(npos[u], lp[e] - us) - 4 * gq;
                } else {
                    // one query: lp[e] is the length (or 0 for an absent head)
#pragma unroll
                    for (int e = 0; e < 2; ++e) lim[u][e] = lp[e] > 0 ? npos[u] - 4 * gq : 0;
                }
            }
            float alpha[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                // v[u][i]: position 4g + i of unit u  (i = 2t + r)
                float v[NU][4];
#pragma unroll
                for (int u = 0; u < NU; ++u) {
                    v[u][0] = x[u][0][0][e]; v[u][1] = x[u][0][1][e];
                    v[u][2] = x[u][1][0][e]; v[u][3] = x[u][1][1][e];
                    if (MODE != PLAIN) {
                        const float tot = col_scan32(v[u], lane);
                        if (MODE == PREFIX) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) v[u][i] += dot_carry[e];
                            dot_carry[e] += tot;
                        }
                    }
                }
                float mx = -INFINITY;
#pragma unroll
                for (int u = 0; u < NU; ++u)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        v[u][i] = i < lim[u][e] ? v[u][i] : -INFINITY;
                        mx = fmaxf(mx, v[u][i]);
                    }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                // scores in log2 units: x * scale_log2 (scale_log2 > 0, so the max
                // of the raw dots scales to the max of the scores)
                const float m_new = fmaxf(m_run[e], mx * A.scale_log2);
                alpha[e] = ex2(m_run[e] - m_new);
                m_run[e] = m_new;
                // every weight (and so the sum and the output) times 2^-wshift:
                // a weight's sum over a group times a V scale then stays inside
                // the fp16 range; out = O / L does not change
                const float m_sh = -m_new - A.wshift;
                float psum = 0.f;
#pragma unroll
                for (int u = 0; u < NU; ++u)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        v[u][i] = ex2(fmaf(v[u][i], A.scale_log2, m_sh));
                        psum += v[u][i];
                    }
                l_run[e] = l_run[e] * alpha[e] + psum;
                // weights that multiply each position's dequantised row
                if (MODE == PREFIX) e_carry[e] *= alpha[e];
#pragma unroll
                for (int u = 0; u < NU; ++u) {
                    float wv[4];
                    if (MODE == SUFFIX) {
                        float pin[4] = {v[u][0], v[u][1], v[u][2], v[u][3]};
                        const float tot = col_scan32(pin, lane);
#pragma unroll
                        for (int i = 0; i < 4; ++i) wv[i] = tot - pin[i] + v[u][i];
                    } else if (MODE == PREFIX) {
                        float pin[4] = {v[u][0], v[u][1], v[u][2], v[u][3]};
                        const float tot = col_scan32(pin, lane);
#pragma unroll
                        for (int i = 0; i < 4; ++i) wv[i] = -(e_carry[e] + pin[i] - v[u][i]);
                        e_carry[e] += tot;
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) wv[i] = v[u][i];
                    }
                    x[u][0][0][e] = wv[0]; x[u][0][1][e] = wv[1];
                    x[u][1][0][e] = wv[2]; x[u][1][1][e] = wv[3];
                }
            }

            // rescale the output accumulators (heads 2tq, 2tq+1), only when a
            // running max moved
            if (__any_sync(0xffffffffu, alpha[0] != 1.0f || alpha[1] != 1.0f)) {
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[mt][0] *= alpha[0]; o[mt][1] *= alpha[1];
                    o[mt][2] *= alpha[0]; o[mt][3] *= alpha[1];
                }
            }

            // ================= V side ======================================
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                const StageMap sm = stage_map<FMT, MODE>(cv.kf, cv.rec_bytes, u);
                v_side<FMT, MODE, ZT, RC>(st, sm, npos[u], first_seg && (MODE != PREFIX || u == 0), gq,
                                      tq, m1024, m64, x[u], o, racc, vkf_keep);
            }

            // PREFIX: close the group (or this range's part of it)
            //   o += W_g (v_f + R_g)
            // where v_f is 0 for a group entered midway (its rows are then
            // relative to the value row before the range's first position)
            if (MODE == PREFIX && last_seg) {
                // a range that ends inside the group hands the next warp the
                // scaled dots of its last position and that position's value row
                const bool hand = (meta.flags & STG_HAND) != 0 &&
                                  range_ok(cv.header, A.hands + HAND_HDR + gw * HANDOFF_FLOATS,
                                           HANDOFF_FLOATS * 4, A.ws, A.ws_floats * 4);
                float *hd = A.hands + HAND_HDR + gw * HANDOFF_FLOATS;
                if (hand && gq == 0) {
                    hd[2 * tq] = dot_carry[0];
                    hd[2 * tq + 1] = dot_carry[1];
                }
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    // RC: R_g of these channels is in the partner thread's
                    // columns 4-7 (lane ^ 2); threads tq >= 2 add e_carry 0
                    const float r_lo = RC ? __shfl_xor_sync(0xffffffffu, o[mt][0], 2) : racc[mt][0];
                    const float r_hi = RC ? __shfl_xor_sync(0xffffffffu, o[mt][2], 2) : racc[mt][2];
                    const float v_lo = h_lo(vkf_keep[mt]) + r_lo;   // channel 16mt+g
                    const float v_hi = h_hi(vkf_keep[mt]) + r_hi;   // channel 16mt+g+8
                    if (hand && tq == 0) {
                        hd[8 + 16 * mt + gq] = v_lo;
                        hd[8 + 16 * mt + gq + 8] = v_hi;
                    }
                    o[mt][0] += e_carry[0] * v_lo; o[mt][1] += e_carry[1] * v_lo;
                    o[mt][2] += e_carry[0] * v_hi; o[mt][3] += e_carry[1] * v_hi;
                    racc[mt][0] = racc[mt][1] = racc[mt][2] = racc[mt][3] = 0.f;
                    if (RC && tq >= 2) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) { e_carry[e] = 0.f; dot_carry[e] = 0.f; }
                if (meta.flags & STG_HEAD) {
                    // a group entered midway has its own record (its scores
                    // lack the dot of the state before it, which the merge
                    // adds); the sequence's record starts afresh
                    write_record(A.heads + gw * PARTIAL_FLOATS);
#pragma unroll
                    for (int e = 0; e < 2; ++e) { m_run[e] = -1e30f; l_run[e] = 0.f; }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
                }
            }
        }

        // ---- release the stage and refill it ------------------------------
        __syncwarp();
        ++consumed;
        if (ic.valid()) {
            if (lane == 0) fence_proxy_async();
            pend = next_stage<FMT, MODE, PAGED>(cv, ic, nvs, A.NHG, mystages + stage_i * STAGE,
                                         mybar + stage_i, mymeta + stage_i, lane, A.fault);
            ++issued;
        }
        stage_i = (stage_i + 1 == NS) ? 0 : stage_i + 1;
    }
    if (cur_b >= 0) flush();

    // A warp that gave up still owns copies in flight: wait for them (bounded)
    // before the CTA can exit and its shared memory be reused.
    if (dead) {
        int si = stage_i;
        for (int k = consumed; k < issued; ++k) {
            if (lane == 0) (void)mbar_wait_bounded(mybar + si, (phase >> si) & 1);
            phase ^= 1u << si;
            si = (si + 1 == NS) ? 0 : si + 1;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// merge: grid (Hq, B), 128 threads (one per channel)
// ---------------------------------------------------------------------------
// merge: grid (nq * Hq, B), 128 threads (one per channel); block x is query
// t = x / Hq, head h = x % Hq, i.e. virtual head t * G + h % G of kv head h / G
// Length decoded for batch entry b: from the stored lengths, or (fused
// append) from the copy the split kernel left in the workspace.
template <bool FIN>
__device__ inline int merge_len(const CacheView &cv, const int32_t *lenv, int b) {
    if constexpr (FIN) return lenv[b];
    else return clamp_len(cv, b);
}

// SEGS (delta format, kf > 32): unit ranges may start and end inside a
// keyframe group (below); wfl holds one flag byte per warp of the sequence.
// BATCH: partial records loaded per round trip.
template <bool FIN, bool SEGS, int BATCH>
__device__ inline void merge_body(const CacheView &cv, int Hq, int G, int NHG, int nq, int64_t NW,
                                  const float *ws, int64_t ws_floats, float *out, uint8_t *wfl) {
    const int t = blockIdx.x / Hq, h = blockIdx.x % Hq, b = blockIdx.y, c = threadIdx.x;
    const int nvs = cv.Hkv * NHG;
    const int32_t *lenv = FIN ? merge_lengths(const_cast<float *>(ws), NW, cv.B * nvs) : nullptr;
    const int len = merge_len<FIN>(cv, lenv, b);
    const int ub = units_of(cv.fmt, cv.kf, len);
    float *dst = out + (((int64_t)b * nq + t) * Hq + h) * D;
    // checked build: this block's output row inside out ([B][nq][Hq][D])
    if (!range_ok(cv.header, dst, D * 4, out, (int64_t)cv.B * nq * Hq * D * 4)) return;
    if (ub == 0) {                      // uniform over the block
        dst[c] = 0.f;
        return;
    }
    const int kvh = h / G, vh = t * G + h % G, hg = vh >> 3, j = vh & 7;
    const int vsl = kvh * NHG + hg;
    // the warps whose unit ranges touch this sequence: found once per block
    __shared__ int64_t sh_w0, sh_w1, sh_total, sh_xs;
    if (threadIdx.x < 32) {
        // units of all batch entries, and of those before b
        int64_t total = 0, mine = 0;
        for (int b0 = 0; b0 < cv.B; b0 += 32) {
            const int xb = b0 + (int)threadIdx.x;
            int64_t u = xb < cv.B ? (int64_t)nvs * units_of(cv.fmt, cv.kf,
                                                            merge_len<FIN>(cv, lenv, xb)) : 0;
            int64_t ub4 = xb < b ? u : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                u += __shfl_xor_sync(0xffffffffu, u, o);
                ub4 += __shfl_xor_sync(0xffffffffu, ub4, o);
            }
            total += u;
            mine += ub4;
        }
        if (threadIdx.x == 0) {
            const int64_t xs = mine + (int64_t)vsl * ub, xe = xs + ub;
            sh_w0 = warp_of(xs, NW, total);
            sh_w1 = warp_of(xe - 1, NW, total);
            sh_total = total;
            sh_xs = xs;
        }
    }
    __syncthreads();
    const int64_t vseq = (int64_t)b * nvs + vsl;
    const int64_t T = sh_total, w0 = sh_w0, w1 = sh_w1, xs = sh_xs, xe = xs + ub;
    // with at least one unit per warp every range is non-empty; otherwise
    // skip the warps that own no unit (they wrote no record)
    const bool dense = T >= NW;
    auto has = [&](int64_t w) {
        return w <= w1 && (dense || range_start(w, NW, T) < range_start(w + 1, NW, T));
    };
    // SEGS: ranges may start and end inside a keyframe group.  A warp that
    // entered a group midway wrote that part as a separate record with scores
    // and value rows relative to the state before its first position; the
    // warp before it handed that state on (absolute, or relative to its own
    // entry state when it too entered the group midway).  Walking the warps
    // in order, the state is carried and each such record made absolute:
    //   m += scaled dot of the state,  o += l * value row of the state.
    // Which warps do what follows from the ranges alone; the flags are worked
    // out once per block, one warp per thread.
    constexpr uint8_t W_ANY = 1, W_HEAD = 2, W_HAND = 4, W_REL = 8;
    const float *heads = nullptr, *hands = nullptr;
    float sl2 = 0.f;
    if constexpr (SEGS) {
        const int spg = seg_per_group(cv.kf);
        for (int64_t k = threadIdx.x; k <= w1 - w0; k += blockDim.x) {
            const int64_t rs = range_start(w0 + k, NW, T), re = range_start(w0 + k + 1, NW, T);
            uint8_t f = 0;
            if (rs < re) {
                f = W_ANY;
                if (rs > xs && (rs - xs) % spg != 0) f |= W_HEAD;
                if (re > xs && re < xe && (re - xs) % spg != 0) f |= W_HAND;
                if ((f & (W_HEAD | W_HAND)) == (W_HEAD | W_HAND) &&
                    (rs - xs) / spg == (re - 1 - xs) / spg)
                    f |= W_REL;
            }
            wfl[k] = f;
        }
        __syncthreads();
        heads = head_records(const_cast<float *>(ws), NW, (int64_t)cv.B * nvs, cv.B);
        hands = handoffs(const_cast<float *>(ws), NW, (int64_t)cv.B * nvs, cv.B);
        // the log2 softmax scale the split kernel used
        sl2 = range_ok(cv.header, hands, 4, ws, ws_floats * 4) ? hands[0] : 0.f;
        hands += HAND_HDR;
    }
    auto flag = [&](int64_t w) -> uint8_t {
        if constexpr (SEGS) return wfl[w - w0];
        else return has(w) ? W_ANY : 0;
    };
    // The sequence's warps in four quarters, one per warp of this block; lane
    // l holds channels 4 l .. 4 l + 3.  The quarters are merged at the end.
    const int wq = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nw = w1 - w0 + 1;
    const int64_t qa = w0 + (nw * wq) / 4, qe = w0 + (nw * (wq + 1)) / 4;
    auto ld4 = [](const float *p) { return *reinterpret_cast<const float4 *>(p); };
    auto fma4 = [](float4 a, float s, float4 c) {
        return make_float4(fmaf(a.x, s, c.x), fmaf(a.y, s, c.y), fmaf(a.z, s, c.z), fmaf(a.w, s, c.w));
    };
    // the carried state (SEGS): head j's scaled dot and this lane's 4 values
    float cdot = 0.f;
    float4 cval = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (SEGS) {
        // entering the quarter inside a group: sum the handoffs back to the
        // nearest absolute one (one step unless warps are shorter than groups)
        if (qa < qe && (flag(qa) & W_HEAD)) {
            for (int64_t k = qa - 1; k >= w0; --k) {
                const uint8_t f = flag(k);
                if (!(f & W_ANY)) continue;
                const float *hh = hands + k * HANDOFF_FLOATS;
                if ((f & W_HAND) && range_ok(cv.header, hh, HANDOFF_FLOATS * 4, ws, ws_floats * 4)) {
                    cdot += hh[j] * sl2;
                    cval = fma4(ld4(hh + 8 + 4 * lane), 1.f, cval);
                }
                if (!(f & W_REL)) break;
            }
        }
    }
    // one pass per quarter, rescaling online: each batch of records moves the
    // running maximum once (records of warps that saw no position carry -1e30)
    float M = -1e30f, L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t w = qa; w < qe; w += BATCH) {
        float mv[BATCH], lv[BATCH], hm[BATCH], hl[BATCH], hdot[BATCH];
        float4 ov[BATCH], ho[BATCH], hval[BATCH];
        uint8_t fl[BATCH];
        bool ok[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            fl[i] = w + i < qe ? flag(w + i) : 0;
            ok[i] = fl[i] & W_ANY;
            const float *rec = ws + (w + i + vseq) * PARTIAL_FLOATS;
            if (DKV_CHECKED && ok[i])
                ok[i] = range_ok(cv.header, rec, PARTIAL_FLOATS * 4, ws, ws_floats * 4);
            mv[i] = ok[i] ? rec[j] : -1e30f;
            lv[i] = ok[i] ? rec[8 + j] : 0.f;
            ov[i] = ok[i] ? ld4(rec + 16 + j * 128 + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (SEGS) {
                const float *hr = heads + (w + i) * PARTIAL_FLOATS;
                const float *hh = hands + (w + i) * HANDOFF_FLOATS;
                const bool hd = (fl[i] & W_HEAD) &&
                                range_ok(cv.header, hr, PARTIAL_FLOATS * 4, ws, ws_floats * 4);
                const bool tl = (fl[i] & W_HAND) &&
                                range_ok(cv.header, hh, HANDOFF_FLOATS * 4, ws, ws_floats * 4);
                if (!hd) fl[i] &= ~W_HEAD;
                if (!tl) fl[i] &= ~W_HAND;
                hm[i] = hd ? hr[j] : -1e30f;
                hl[i] = hd ? hr[8 + j] : 0.f;
                ho[i] = hd ? ld4(hr + 16 + j * 128 + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
                hdot[i] = tl ? hh[j] * sl2 : 0.f;
                hval[i] = tl ? ld4(hh + 8 + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        if constexpr (SEGS) {
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                if (fl[i] & W_HEAD) {
                    hm[i] += cdot;
                    ho[i] = fma4(cval, hl[i], ho[i]);
                }
                if (fl[i] & W_HAND) {
                    const bool rel = fl[i] & W_REL;
                    cdot = rel ? cdot + hdot[i] : hdot[i];
                    cval = rel ? fma4(hval[i], 1.f, cval) : hval[i];
                }
            }
        }
        float Mn = M;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            Mn = fmaxf(Mn, mv[i]);
            if constexpr (SEGS) Mn = fmaxf(Mn, hm[i]);
        }
        const float sc = exp2f(M - Mn);
        L *= sc;
        O = make_float4(O.x * sc, O.y * sc, O.z * sc, O.w * sc);
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const float e = exp2f(mv[i] - Mn);
            L = fmaf(lv[i], e, L);
            O = fma4(ov[i], e, O);
            if constexpr (SEGS) {
                const float eh = exp2f(hm[i] - Mn);
                L = fmaf(hl[i], eh, L);
                O = fma4(ho[i], eh, O);
            }
        }
        M = Mn;
    }
    // merge the four quarters (log-sum-exp), one channel per thread
    __shared__ float q_m[4], q_l[4];
    __shared__ float4 q_o[4][32];
    if (lane == 0) { q_m[wq] = M; q_l[wq] = L; }
    q_o[wq][lane] = O;
    __syncthreads();
    float Mx = q_m[0];
#pragma unroll
    for (int q = 1; q < 4; ++q) Mx = fmaxf(Mx, q_m[q]);
    float Lt = 0.f, Ot = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float e = exp2f(q_m[q] - Mx);
        const float4 v = q_o[q][c >> 2];
        const float oc = (c & 3) == 0 ? v.x : (c & 3) == 1 ? v.y : (c & 3) == 2 ? v.z : v.w;
        Lt = fmaf(q_l[q], e, Lt);
        Ot = fmaf(oc, e, Ot);
    }
    dst[c] = Lt > 0.f ? Ot / Lt : 0.f;  // a causal query with no position gets 0
}

template <bool FIN, bool SEGS, int BATCH>
__device__ inline void merge_entry(const CacheView &cv, int Hq, int G, int NHG, int nq, int64_t NW,
                                   const float *ws, int64_t ws_floats, float *out) {
    extern __shared__ uint8_t merge_flags[];        // SEGS: one byte per warp slot
    pdl_trigger();
    pdl_wait();                                     // the split kernel's records
    merge_body<FIN, SEGS, BATCH>(cv, Hq, G, NHG, nq, NW, ws, ws_floats, out, merge_flags);
    if constexpr (FIN) {
        // fused append: publish batch entry b's new length (no other block of
        // this launch reads it) and make the state slot the split kernel
        // wrote current
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            int l;
            if (takes_append(cv, blockIdx.y, l)) cv.seqlen[blockIdx.y] = l + cv.len_add;
            if (blockIdx.y == 0) cv.header[2] ^= 1;
        }
    }
}

template <bool FIN, bool SEGS, int BATCH>
__global__ void __launch_bounds__(128) merge_kernel(CacheView cv, int Hq, int G, int NHG, int nq,
                                                    int64_t NW, const float *ws, int64_t ws_floats,
                                                    float *out) {
    merge_entry<FIN, SEGS, BATCH>(cv, Hq, G, NHG, nq, NW, ws, ws_floats, out);
}

// The whole-group merge capped at 72 registers, so that 7 blocks fit an SM
// instead of 6.  It is taken when the grid is more than one wave of the
// uncapped kernel (a batch of 16 x 64 query heads: 1024 blocks, 1.15 waves
// uncapped, 0.99 capped); smaller grids keep the uncapped kernel, which does
// not spill.
template <bool FIN, int BATCH>
__global__ void __launch_bounds__(128, 7) merge_kernel_capped(CacheView cv, int Hq, int G, int NHG,
                                                              int nq, int64_t NW, const float *ws,
                                                              int64_t ws_floats, float *out) {
    merge_entry<FIN, false, BATCH>(cv, Hq, G, NHG, nq, NW, ws, ws_floats, out);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int FMT, int MODE>
static size_t split_smem() {
    return (size_t)SmemMap<FMT, MODE>::BYTES;
}

// Per-device host state of the launches (the persistent grid of an instance,
// whether an instance's shared-memory attribute is set), shared by every host
// thread: read lock-free once published, computed under a mutex.
constexpr int kMaxDevices = 64;
static std::mutex g_launch_mu;

static cudaError_t current_device(int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    return (*dev < 0 || *dev >= kMaxDevices) ? cudaErrorInvalidDevice : cudaSuccess;
}

// how many blocks of the uncapped whole-group merge the current device holds
// at once (resident blocks per SM x SMs), cached per device
static cudaError_t merge_wave(int64_t *blocks) {
    static std::atomic<int64_t> wave_of[kMaxDevices];  // 0: not queried yet
    int dev;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    int64_t w = wave_of[dev].load(std::memory_order_acquire);
    if (w == 0) {
        int per_sm = 0, nsm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, merge_kernel<false, false, DKV_MERGE_BATCH>, 128, 0);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        w = (int64_t)(per_sm < 1 ? 1 : per_sm) * nsm;
        wave_of[dev].store(w, std::memory_order_release);
    }
    *blocks = w;
    return cudaSuccess;
}

template <int FMT, int MODE, bool ZT>
static cudaError_t geom_for(SplitGeom *g) {
    static std::atomic<int> ctas_of[kMaxDevices];      // 0: not computed yet
    int dev;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    int ctas = ctas_of[dev].load(std::memory_order_acquire);
    if (ctas == 0) {
        std::lock_guard<std::mutex> lock(g_launch_mu);
        ctas = ctas_of[dev].load(std::memory_order_relaxed);
        if (ctas == 0) {
            const size_t sm = split_smem<FMT, MODE>();
            e = cudaFuncSetAttribute(split_kernel<FMT, MODE, ZT, false, false, false, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e != cudaSuccess) return e;
            int per_sm = 0, nsm = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, split_kernel<FMT, MODE, ZT, false, false, false, false>, WARPS * 32, sm);
            if (e != cudaSuccess) return e;
            e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            ctas = (per_sm < 1 ? 1 : per_sm) * nsm;
            ctas_of[dev].store(ctas, std::memory_order_release);
        }
    }
    g->ctas = ctas;
    g->warps_per_cta = WARPS;
    return cudaSuccess;
}

// The kernel instance for a cache: format, mode (kf <= 32: whole groups per
// unit; kf > 32: 32-position segments) and whether tail slots need their
// scales zeroed (kf != 32 for the delta format).  The persistent grid fills
// the GPU, but never gives a warp fewer than kMinUnitsPerWarp of the most
// units the cache can hold (max_units), so a small cache is not spread over
// warps that would own nothing (the merge walks the warps of a sequence).
// The merge and the workspace size derive the warp count the same way.
constexpr int64_t kMinUnitsPerWarp = 4;

static void clamp_geometry(SplitGeom *g, int64_t max_units) {
    const int64_t want = (max_units + kMinUnitsPerWarp * WARPS - 1) / (kMinUnitsPerWarp * WARPS);
    if (want < g->ctas) g->ctas = (int)(want < 1 ? 1 : want);
}

cudaError_t split_geometry(int fmt, int kf, int64_t max_units, SplitGeom *g) {
    cudaError_t e;
    if (fmt == DKV_FMT_DELTA) {
        if (kf == SEG) e = geom_for<DKV_FMT_DELTA, SUFFIX, false>(g);
        else e = kf < SEG ? geom_for<DKV_FMT_DELTA, SUFFIX, true>(g)
                          : geom_for<DKV_FMT_DELTA, PREFIX, true>(g);
    } else if (fmt == DKV_FMT_Q4_0) {
        e = geom_for<DKV_FMT_Q4_0, PLAIN, false>(g);
    } else {
        e = geom_for<DKV_FMT_FP16, PLAIN, false>(g);
    }
    if (e == cudaSuccess) clamp_geometry(g, max_units);
    return e;
}

// Units the split kernel can see for a cache: every sequence (b, kv head,
// head group) at capacity.
int64_t split_max_units(int fmt, int kf, int B, int Hkv, int nhg, int cap) {
    return (int64_t)B * Hkv * nhg * units_of(fmt, fmt == DKV_FMT_DELTA ? kf : 1, cap);
}

// Every instance runs on the contiguous one-query instance's grid (the merge
// and the workspace size follow that grid); a persistent grid is correct at
// any size.
template <int FMT, int MODE, bool ZT, bool PAGED, bool MQ, bool APP, bool QHL, bool RC = false>
static cudaError_t launch_inst(const SplitArgs &a, int ctas, cudaStream_t st) {
    if (PAGED || MQ || APP || QHL || RC) {
        static std::atomic<bool> set_on[kMaxDevices];   // per instance and device
        int dev;
        cudaError_t e = current_device(&dev);
        if (e != cudaSuccess) return e;
        if (!set_on[dev].load(std::memory_order_acquire)) {
            std::lock_guard<std::mutex> lock(g_launch_mu);
            if (!set_on[dev].load(std::memory_order_relaxed)) {
                e = cudaFuncSetAttribute(split_kernel<FMT, MODE, ZT, PAGED, MQ, APP, QHL, RC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)split_smem<FMT, MODE>());
                if (e != cudaSuccess) return e;
                set_on[dev].store(true, std::memory_order_release);
            }
        }
    }
    return launch_pdl(split_kernel<FMT, MODE, ZT, PAGED, MQ, APP, QHL, RC>, dim3(ctas),
                      dim3(WARPS * 32), split_smem<FMT, MODE>(), st, a);
}

// fp32 queries take the hi + lo instance
template <int FMT, int MODE, bool ZT, bool PAGED, bool MQ, bool APP>
static cudaError_t launch_q(const SplitArgs &a, int ctas, cudaStream_t st) {
    return a.q_dtype == DKV_F32 ? launch_inst<FMT, MODE, ZT, PAGED, MQ, APP, true>(a, ctas, st)
                                : launch_inst<FMT, MODE, ZT, PAGED, MQ, APP, false>(a, ctas, st);
}

template <int FMT, int MODE, bool ZT>
static cudaError_t launch_split_t(const SplitArgs &a_in, cudaStream_t st) {
    SplitGeom g;
    cudaError_t e = geom_for<FMT, MODE, ZT>(&g);
    if (e != cudaSuccess) return e;
    clamp_geometry(&g, split_max_units(a_in.cv.fmt, a_in.cv.kf, a_in.cv.B, a_in.cv.Hkv, a_in.NHG,
                                       a_in.cv.cap));
    SplitArgs a = a_in;
    {
        const int64_t NW = (int64_t)g.ctas * g.warps_per_cta;
        const int64_t nseq = (int64_t)a.cv.B * a.cv.Hkv * a.NHG;
        a.heads = head_records(a.ws, NW, nseq, a.cv.B);
        a.hands = handoffs(a.ws, NW, nseq, a.cv.B);
    }
    const bool paged = a.cv.pg != 0, mq = a.nq > 1, app = a.cv.len_add > 0;
    if (!paged && !mq && !app) {
        // kf > 32 with at most 4 heads per kv head: R_g in the spare columns
        if constexpr (FMT == DKV_FMT_DELTA && MODE == PREFIX)
            if (a.G <= 4 && a.q_dtype != DKV_F32)
                return launch_inst<FMT, MODE, ZT, false, false, false, false, true>(a, g.ctas, st);
        return launch_q<FMT, MODE, ZT, false, false, false>(a, g.ctas, st);
    }
    if constexpr (FMT == DKV_FMT_DELTA) {        // only the delta format pages / takes queries
        if (app) {
            if (paged && mq) return launch_q<FMT, MODE, ZT, true, true, true>(a, g.ctas, st);
            if (paged) return launch_q<FMT, MODE, ZT, true, false, true>(a, g.ctas, st);
            if (mq) return launch_q<FMT, MODE, ZT, false, true, true>(a, g.ctas, st);
            return launch_q<FMT, MODE, ZT, false, false, true>(a, g.ctas, st);
        }
        if (paged && mq) return launch_q<FMT, MODE, ZT, true, true, false>(a, g.ctas, st);
        if (paged) return launch_q<FMT, MODE, ZT, true, false, false>(a, g.ctas, st);
        return launch_q<FMT, MODE, ZT, false, true, false>(a, g.ctas, st);
    } else {
        return cudaErrorInvalidValue;
    }
}

cudaError_t launch_split(const CacheView &cv, const void *Q, int q_dtype, int Hq, int nq,
                         float softmax_scale, float *ws, int64_t ws_floats, int fault,
                         cudaStream_t st, const void *K_new, const void *V_new, int kv_dtype) {
    SplitArgs a;
    a.fault = fault == 1 ? 1 : 0;
    // test support (mode 2): the workspace declared two records short
    a.ws_floats = fault == 2 ? ws_floats - 2 * PARTIAL_FLOATS : ws_floats;
    a.Kn = K_new;
    a.Vn = V_new;
    a.kv_dtype = kv_dtype;
    a.cv = cv;
    a.Q = Q;
    a.q_dtype = q_dtype;
    a.Hq = Hq;
    a.G = Hq / cv.Hkv;
    a.nq = nq;
    a.NHG = (nq * a.G + 7) / 8;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    // weight scaling: 2^-ceil(log2 kf) for the delta format (a weight sum over
    // a group is at most kf), none for the comparators (one token per row)
    a.wshift = 0.f;
    if (cv.fmt == DKV_FMT_DELTA) {
        int sh = 0;
        while ((1 << sh) < cv.kf && sh < 24) ++sh;
        a.wshift = (float)sh;
    }
    a.ws = ws;
    if (cv.fmt == DKV_FMT_DELTA) {
        if (cv.kf == SEG) return launch_split_t<DKV_FMT_DELTA, SUFFIX, false>(a, st);
        return cv.kf < SEG ? launch_split_t<DKV_FMT_DELTA, SUFFIX, true>(a, st)
                           : launch_split_t<DKV_FMT_DELTA, PREFIX, true>(a, st);
    }
    if (cv.fmt == DKV_FMT_Q4_0) return launch_split_t<DKV_FMT_Q4_0, PLAIN, false>(a, st);
    return launch_split_t<DKV_FMT_FP16, PLAIN, false>(a, st);
}

cudaError_t launch_merge(const CacheView &cv, int Hq, int nq, float *out, const float *ws,
                         int64_t ws_floats, cudaStream_t st) {
    const int G = Hq / cv.Hkv;
    const int NHG = (nq * G + 7) / 8;
    SplitGeom g;
    cudaError_t e = split_geometry(cv.fmt, cv.kf, split_max_units(cv.fmt, cv.kf, cv.B, cv.Hkv, NHG,
                                                                  cv.cap), &g);
    if (e != cudaSuccess) return e;
    dim3 grid(nq * Hq, cv.B);
    const int64_t NW = (int64_t)g.ctas * g.warps_per_cta;
    if (cv.fmt == DKV_FMT_DELTA && cv.kf > SEG) {
        // a flag byte for each warp slot a sequence can span
        const size_t fl = (size_t)(NW + 15) / 16 * 16;
        if (fl > 48 * 1024) return cudaErrorInvalidConfiguration;
        if (cv.len_add > 0)
            e = launch_pdl(merge_kernel<true, true, DKV_MERGE_BATCH>, grid, dim3(128), fl, st,
                           cv, Hq, G, NHG, nq, NW, (const float *)ws, ws_floats, out);
        else
            e = launch_pdl(merge_kernel<false, true, DKV_MERGE_BATCH>, grid, dim3(128), fl, st,
                           cv, Hq, G, NHG, nq, NW, (const float *)ws, ws_floats, out);
    } else {
        int64_t wave = 0;
        e = merge_wave(&wave);
        if (e != cudaSuccess) return e;
        const bool cap = (int64_t)grid.x * grid.y > wave;
        if (cv.len_add > 0)
            e = cap ? launch_pdl(merge_kernel_capped<true, DKV_MERGE_BATCH>, grid, dim3(128), 0,
                                 st, cv, Hq, G, NHG, nq, NW, (const float *)ws, ws_floats, out)
                    : launch_pdl(merge_kernel<true, false, DKV_MERGE_BATCH>, grid, dim3(128), 0, st,
                                 cv, Hq, G, NHG, nq, NW, (const float *)ws, ws_floats, out);
        else
            e = cap ? launch_pdl(merge_kernel_capped<false, DKV_MERGE_BATCH>, grid, dim3(128), 0,
                                 st, cv, Hq, G, NHG, nq, NW, (const float *)ws, ws_floats, out)
                    : launch_pdl(merge_kernel<false, false, DKV_MERGE_BATCH>, grid, dim3(128), 0, st,
                                 cv, Hq, G, NHG, nq, NW, (const float *)ws, ws_floats, out);
    }
    return e;
}

}  // namespace dkv
