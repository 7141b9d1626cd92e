/*
 * dkv_oracle.c -- plain, slow, obviously-correct CPU oracle for the Delta-KV
 * decode path.  TEST INFRASTRUCTURE ONLY: it exists so the CUDA library can be
 * checked against an independent statement of the method.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline / reference legs may
 * load it; the product path never does.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Sources (web pages; cited by page title and section):
 *  [DKV]  "영상 압축 기법을 KV 캐시에 적용해 Q4 양자화 오차를 10,000배 줄인
 *          Delta-KV" (jeff.news, article 892).
 *          section "핵심 아이디어": a keyframe is stored, then only the
 *          token-to-token differences, quantised to 4 bits like Q4_0 does for
 *          absolute values.
 *          section "벤치마크": keyframe interval kf (kf=32), Q4_0 and F16
 *          caches as the comparators.
 *          section "컨텍스트 길이에 따른 안정성": no error blow-up even with
 *          512 delta frames between keyframes (read here as: the delta is taken
 *          against the *reconstructed* previous token -- closed loop).
 *  [VQ]   "KV 캐시 벡터 양자화와 주의 보존 변환" (llm-wiki.hwlabs.dev),
 *          section "KV 캐시가 왜 병목인가": one decode step loads every previous
 *          K/V, forms QK^T, applies softmax and aggregates A.V.
 *
 * The Q4_0 block rule used by both quantised formats: blocks of 32 elements,
 * m = the signed element of largest magnitude, d = m / -8 stored as fp16,
 * code = min(15, trunc(x/d + 8.5)), dequantised value (code - 8) * d.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - keyframe positions are p mod kf == 0, per sequence, from position 0;
 *  - the quantiser divides by the *stored* fp16 scale d16 (as fp32), with an
 *    IEEE correctly-rounded fp32 division, then adds 8.5f in fp32;
 *  - ties in |m| go to the lowest index;
 *  - d16 == +-0 (all-zero block or underflow) gives code 8 everywhere;
 *  - the code is clamped to [0, 15] (the lower clamp only matters when the
 *    fp16 rounding of a subnormal scale shrinks |d16| below |m/8|);
 *  - the reconstruction state is fp32 and strictly sequential.
 *
 * Floating point: every quantiser step is a single IEEE binary32 operation in
 * source order (build with -ffp-contract=off, no fast-math); attention is
 * carried out in binary64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define OR_BLOCK 32

/* ---------------------------------------------------------------------------
 * IEEE 754 binary16 <-> binary32, written from the format definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits; subnormals;
 * round to nearest, ties to even).
 * ------------------------------------------------------------------------- */
float or_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);              /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);  /* (1.f) * 2^(e-15) */
    return (float)(sign ? -v : v);
}

uint16_t or_f32_to_f16(float x)
{
    uint32_t bits;
    memcpy(&bits, &x, 4);
    uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
    double a = fabs((double)x);
    if (isnan(x)) return (uint16_t)(sign | 0x7e00u);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);  /* rounds to inf */
    /* Express a as an integer multiple of the binary16 spacing at its
     * exponent, rounding the multiple to nearest even. */
    int e;
    double frac = frexp(a, &e);          /* a = frac * 2^e, frac in [0.5,1) */
    (void)frac;
    int exp16 = e - 1;                   /* a in [2^exp16, 2^(exp16+1)) */
    if (a == 0.0) return sign;
    if (exp16 < -14) exp16 = -14;        /* subnormal range: spacing 2^-24 */
    double ulp = ldexp(1.0, exp16 - 10);
    double q = a / ulp;                  /* exact: power-of-two scaling */
    double r = floor(q);
    double rem = q - r;
    if (rem > 0.5 || (rem == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double v = r * ulp;                  /* rounded magnitude */
    if (v >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    /* Re-encode v. */
    if (v < ldexp(1.0, -14)) {           /* subnormal (or zero) */
        return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24)));
    }
    int ev;
    frexp(v, &ev);
    int E = ev - 1;                      /* v in [2^E, 2^(E+1)) */
    int mant = (int)(v / ldexp(1.0, E - 10)) - 1024;
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)mant);
}

/* ---------------------------------------------------------------------------
 * Q4_0 block quantiser on 32 fp32 values.
 * ------------------------------------------------------------------------- */
void or_quant_block(const float *v, uint16_t *d16_out, uint8_t *codes)
{
    /* m: the signed element of largest magnitude, lowest index on ties. */
    int arg = 0;
    float best = fabsf(v[0]);
    for (int i = 1; i < OR_BLOCK; ++i) {
        float a = fabsf(v[i]);
        if (a > best) { best = a; arg = i; }
    }
    float m = v[arg];
    float d32 = m / -8.0f;
    uint16_t d16 = or_f32_to_f16(d32);
    float d = or_f16_to_f32(d16);
    *d16_out = d16;
    for (int i = 0; i < OR_BLOCK; ++i) {
        int c;
        if (d == 0.0f) {
            c = 8;
        } else {
            float t = v[i] / d;          /* IEEE binary32 division */
            float u = t + 8.5f;          /* binary32 add */
            c = (int)truncf(u);
            if (c > 15) c = 15;
            if (c < 0) c = 0;
        }
        codes[i] = (uint8_t)c;
    }
}

/* Dequantised value of one code under scale bits d16: (code - 8) * d. */
static float or_dequant(uint8_t code, uint16_t d16)
{
    float d = or_f16_to_f32(d16);
    float step = (float)((int)code - 8) * d;  /* exact: 4-bit x 11-bit */
    return step;
}

/* ---------------------------------------------------------------------------
 * Delta-KV encoder, one sequence of one tensor (K or V), positions
 * [start, start+n).  Arrays are indexed by absolute position:
 *   x      [n][D]         input values of the new positions (fp32)
 *   kfr    [ng][D]        fp16 bits of the keyframes (group g at row g)
 *   scales [cap][D/32]    fp16 bits of the delta scales (keyframe rows untouched)
 *   codes  [cap][D]       codes 0..15 (keyframe rows untouched)
 *   xhat   [cap][D]       reconstruction (may be NULL)
 *   state  [D]            in: x^ of position start-1 (ignored when start is a
 *                         keyframe position); out: x^ of position start+n-1
 * ------------------------------------------------------------------------- */
void or_delta_encode_range(int start, int n, int D, int kf, const float *x,
                           uint16_t *kfr, uint16_t *scales, uint8_t *codes,
                           float *xhat, float *state)
{
    const int nb = D / OR_BLOCK;
    float delta[OR_BLOCK];
    for (int i = 0; i < n; ++i) {
        int p = start + i;
        const float *xp = x + (size_t)i * D;
        if (p % kf == 0) {
            /* keyframe: fp16 of the value; x^ = that fp16 value */
            int g = p / kf;
            for (int c = 0; c < D; ++c) {
                uint16_t h = or_f32_to_f16(xp[c]);
                kfr[(size_t)g * D + c] = h;
                state[c] = or_f16_to_f32(h);
            }
        } else {
            for (int b = 0; b < nb; ++b) {
                for (int j = 0; j < OR_BLOCK; ++j) {
                    int c = b * OR_BLOCK + j;
                    delta[j] = xp[c] - state[c];   /* x_t - x^_{t-1} */
                }
                uint16_t d16;
                uint8_t cb[OR_BLOCK];
                or_quant_block(delta, &d16, cb);
                scales[(size_t)p * nb + b] = d16;
                for (int j = 0; j < OR_BLOCK; ++j) {
                    int c = b * OR_BLOCK + j;
                    codes[(size_t)p * D + c] = cb[j];
                    state[c] = state[c] + or_dequant(cb[j], d16);  /* closed loop */
                }
            }
        }
        if (xhat)
            memcpy(xhat + (size_t)p * D, state, sizeof(float) * D);
    }
}

/* Reconstruct positions [0, T) of one Delta-KV tensor from its stored codes,
 * scales and keyframes alone (the decoder side of the scheme). */
void or_delta_decode(int T, int D, int kf, const uint16_t *kfr,
                     const uint16_t *scales, const uint8_t *codes, float *xhat)
{
    const int nb = D / OR_BLOCK;
    float *cur = (float *)malloc(sizeof(float) * D);
    for (int p = 0; p < T; ++p) {
        if (p % kf == 0) {
            for (int c = 0; c < D; ++c)
                cur[c] = or_f16_to_f32(kfr[(size_t)(p / kf) * D + c]);
        } else {
            for (int c = 0; c < D; ++c)
                cur[c] = cur[c] + or_dequant(codes[(size_t)p * D + c],
                                             scales[(size_t)p * nb + c / OR_BLOCK]);
        }
        memcpy(xhat + (size_t)p * D, cur, sizeof(float) * D);
    }
    free(cur);
}

/* Plain Q4_0 comparator: the same block rule on the values themselves. */
void or_q4_encode(int T, int D, const float *x, uint16_t *scales, uint8_t *codes,
                  float *xhat)
{
    const int nb = D / OR_BLOCK;
    for (int p = 0; p < T; ++p) {
        for (int b = 0; b < nb; ++b) {
            const float *v = x + (size_t)p * D + b * OR_BLOCK;
            uint16_t d16;
            or_quant_block(v, &d16, codes + (size_t)p * D + b * OR_BLOCK);
            scales[(size_t)p * nb + b] = d16;
            if (xhat)
                for (int j = 0; j < OR_BLOCK; ++j)
                    xhat[(size_t)p * D + b * OR_BLOCK + j] =
                        or_dequant(codes[(size_t)p * D + b * OR_BLOCK + j], d16);
        }
    }
}

/* F16 comparator: each value rounded to binary16. */
void or_f16_encode(int T, int D, const float *x, uint16_t *out, float *xhat)
{
    for (size_t i = 0; i < (size_t)T * D; ++i) {
        out[i] = or_f32_to_f16(x[i]);
        if (xhat) xhat[i] = or_f16_to_f32(out[i]);
    }
}

/* ---------------------------------------------------------------------------
 * One decode step of attention for the G query heads that share one KV head,
 * brute force in binary64 ([VQ] "KV 캐시가 왜 병목인가": QK^T, softmax, A.V):
 *   s_p = scale * sum_c q[c] * k^_p[c]
 *   w_p = exp(s_p - max_p s_p) / sum_p exp(s_p - max_p s_p)
 *   o[c] = sum_p w_p * v^_p[c]
 *   q [G][D] (binary64), khat/vhat [T][D] (binary32), out [G][D] (binary64).
 *   T == 0 gives o = 0.
 * ------------------------------------------------------------------------- */
void or_attn(int T, int D, int G, const double *q, const float *khat,
             const float *vhat, double scale, double *out)
{
    double *s = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
    for (int h = 0; h < G; ++h) {
        const double *qh = q + (size_t)h * D;
        double mx = -INFINITY;
        for (int p = 0; p < T; ++p) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c)
                acc += qh[c] * (double)khat[(size_t)p * D + c];
            s[p] = scale * acc;
            if (s[p] > mx) mx = s[p];
        }
        double den = 0.0;
        for (int p = 0; p < T; ++p) {
            s[p] = exp(s[p] - mx);
            den += s[p];
        }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int p = 0; p < T; ++p)
                acc += s[p] * (double)vhat[(size_t)p * D + c];
            out[(size_t)h * D + c] = T > 0 ? acc / den : 0.0;
        }
    }
    free(s);
}

/* ---------------------------------------------------------------------------
 * Long-range reference encoder (the training-free part of DeltaKV), one
 * sequence of one tensor.  Source: the gist.science summary of DeltaKV
 * (arXiv 2602.08005):
 *   section "2. 핵심 관찰": similar tokens are spread far apart over the
 *     context (long-range inter-token similarity);
 *   section "A. DeltaKV 프레임워크": "Strided Reference Selection" (the
 *     reference set is the tokens at a fixed stride), "Residual Encoding"
 *     (subtract the mean of the most similar reference tokens; encode the
 *     residual), "Reconstruction" (add that mean back);
 *   section "4. 주요 기여 및 결과", "양자화 친화성": the residuals sit near
 *     zero and take 4-bit quantisation.
 * The learned compressor is replaced by the Q4_0 block rule.
 * Readings where the page is silent:
 *   - the references are the positions r with r mod s == 0, stored as fp16;
 *   - token p (not a reference) chooses among the references before it, r < p;
 *   - "most similar" is the smallest squared Euclidean distance to the stored
 *     reference, summed over channels c = 0 .. D-1 in binary64, in that order
 *     (each difference, square and sum one binary64 operation); ties go to
 *     the smaller position;
 *   - the m most similar are used (all of them when fewer exist); their mean
 *     is the binary32 sum in ascending position, divided (binary32) by their
 *     count;
 *   - the residual x_p - mean (binary32) is quantised with the Q4_0 block
 *     rule and x^_p = mean + (code - 8) * d.
 * Outputs, indexed by position p in [0, T):
 *   ref    [T][m]   reference numbers r / s of the chosen references in
 *                   ascending order; -1 for unused slots and reference tokens
 *   kfr    [ng][D]  fp16 bits of reference g (position g * s), ng = ceil(T/s)
 *   scales [T][D/32], codes [T][D]  (zero on reference rows)
 *   xhat   [T][D]   reconstruction
 * ------------------------------------------------------------------------- */
void or_lr_encode(int T, int D, int s, int m, const float *x, int32_t *ref, uint16_t *kfr,
                  uint16_t *scales, uint8_t *codes, float *xhat)
{
    const int nb = D / OR_BLOCK;
    const int ng = (T + s - 1) / s;
    float *kv = (float *)malloc(sizeof(float) * (size_t)(ng > 0 ? ng : 1) * D);
    double *dist = (double *)malloc(sizeof(double) * (size_t)(ng > 0 ? ng : 1));
    int *sel = (int *)malloc(sizeof(int) * (size_t)m);
    float *mean = (float *)malloc(sizeof(float) * (size_t)D);
    float res[OR_BLOCK];
    for (int p = 0; p < T; ++p) {
        const float *xp = x + (size_t)p * D;
        for (int k = 0; k < m; ++k) ref[(size_t)p * m + k] = -1;
        memset(scales + (size_t)p * nb, 0, sizeof(uint16_t) * (size_t)nb);
        memset(codes + (size_t)p * D, 0, (size_t)D);
        if (p % s == 0) {                    /* a reference token: fp16 */
            const int g = p / s;
            for (int c = 0; c < D; ++c) {
                uint16_t h = or_f32_to_f16(xp[c]);
                kfr[(size_t)g * D + c] = h;
                kv[(size_t)g * D + c] = or_f16_to_f32(h);
                xhat[(size_t)p * D + c] = kv[(size_t)g * D + c];
            }
            continue;
        }
        const int nc = (p - 1) / s + 1;      /* references 0, s, 2s, ... below p */
        for (int g = 0; g < nc; ++g) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c) {
                double diff = (double)xp[c] - (double)kv[(size_t)g * D + c];
                double sq = diff * diff;
                acc = acc + sq;
            }
            dist[g] = acc;
        }
        const int me = nc < m ? nc : m;
        for (int k = 0; k < me; ++k) {       /* k-th smallest, smaller position first */
            int best = -1;
            for (int g = 0; g < nc; ++g) {
                int used = 0;
                for (int j = 0; j < k; ++j) used |= (sel[j] == g);
                if (used) continue;
                if (best < 0 || dist[g] < dist[best]) best = g;
            }
            sel[k] = best;
        }
        for (int i = 1; i < me; ++i)         /* ascending position */
            for (int j = i; j > 0 && sel[j - 1] > sel[j]; --j) {
                int t = sel[j]; sel[j] = sel[j - 1]; sel[j - 1] = t;
            }
        for (int k = 0; k < me; ++k) ref[(size_t)p * m + k] = sel[k];
        for (int c = 0; c < D; ++c) {
            float acc = 0.0f;
            for (int k = 0; k < me; ++k) acc = acc + kv[(size_t)sel[k] * D + c];
            mean[c] = acc / (float)me;
        }
        for (int b = 0; b < nb; ++b) {
            for (int i = 0; i < OR_BLOCK; ++i)
                res[i] = xp[b * OR_BLOCK + i] - mean[b * OR_BLOCK + i];
            uint16_t d16;
            uint8_t *cb = codes + (size_t)p * D + b * OR_BLOCK;
            or_quant_block(res, &d16, cb);
            scales[(size_t)p * nb + b] = d16;
            for (int i = 0; i < OR_BLOCK; ++i)
                xhat[(size_t)p * D + b * OR_BLOCK + i] =
                    mean[b * OR_BLOCK + i] + or_dequant(cb[i], d16);
        }
    }
    free(kv);
    free(dist);
    free(sel);
    free(mean);
}
