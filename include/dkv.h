/*
 * dkv.h -- C ABI of the Delta-KV decode library for NVIDIA B200 (sm_100a).
 *
 * A Delta-KV cache stores every kf-th token of each (batch, kv-head)
 * sequence as an fp16 keyframe and every other token as a 4-bit, Q4_0-style
 * quantised difference against the reconstructed previous token (closed
 * loop).  Sources:
 *   page "영상 압축 기법을 KV 캐시에 적용해 Q4 양자화 오차를 10,000배 줄인
 *   Delta-KV" (jeff.news article 892): section "핵심 아이디어" (keyframe +
 *   4-bit token-to-token differences instead of absolute values), section
 *   "벤치마크" (kf = 32; Q4_0 and F16 caches as comparators), section
 *   "컨텍스트 길이에 따른 안정성" (no error build-up with 512 delta frames);
 *   page "KV 캐시 벡터 양자화와 주의 보존 변환" (llm-wiki), section
 *   "KV 캐시가 왜 병목인가" (a decode step reads every cached K/V from HBM,
 *   forms QK^T, softmax and A.V; the read is the bottleneck).
 *
 * The Q4_0 block rule (both quantised formats): blocks of 32 channels;
 * m = signed element of largest |.| (lowest index on ties); d = fp16(m / -8);
 * code = clamp(trunc(x / d + 8.5), 0, 15) with an IEEE fp32 division by the
 * stored fp16 d; d == 0 gives code 8; dequantised value (code - 8) * d.
 *
 * Conventions for every entry point:
 *  - The caller owns all memory.  The library never allocates, never frees
 *    and never synchronises, except dkv_get_device_status (which synchronises
 *    the stream it is given).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream.  The append,
 *    decode-split and merge kernels, and the long-range decode's kernels, are
 *    launched with programmatic stream serialization: one may be scheduled
 *    while the kernel before it on the stream is finishing, but it waits for
 *    that kernel to complete before its first global memory access, so stream
 *    order holds for all memory.
 *  - Host-side validation happens before any launch; a failed check returns
 *    an error and launches nothing.  Device pointers must be 16-byte aligned
 *    (DKV_EALIGN otherwise); the cache base must be 256-byte aligned.
 *  - Faults found on the device (a sequence length out of range, an append
 *    past capacity, a pipeline wait that ran out) set a status word inside
 *    the cache; the kernel skips the affected work and returns.  Nothing
 *    traps and nothing waits without a bound.  Read and clear the word with
 *    dkv_get_device_status.
 *  - head_dim must be 128.  Query head h reads KV head h / (Hq / Hkv).
 *  - Inputs must be finite and within the fp16 range.
 */
#ifndef DKV_H
#define DKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DKV_ABI_VERSION 3

typedef enum {
    DKV_OK = 0,
    DKV_EINVAL = 1,        /* bad argument: null pointer, bad shape, bad enum */
    DKV_EALIGN = 2,        /* pointer not aligned as required */
    DKV_ECAPACITY = 3,     /* request exceeds cache capacity or workspace size */
    DKV_EUNSUPPORTED = 4,  /* valid but not supported (e.g. head_dim != 128) */
    DKV_ECUDA = 5,         /* a CUDA runtime call or launch failed */
    DKV_EDEVICE = 6        /* the device status word is non-zero */
} dkv_status;

typedef enum {
    DKV_FMT_FP16 = 0,      /* comparator: fp16 values */
    DKV_FMT_Q4_0 = 1,      /* comparator: Q4_0 on absolute values */
    DKV_FMT_DELTA = 2      /* keyframe + closed-loop 4-bit deltas */
} dkv_format;

typedef enum { DKV_F32 = 0, DKV_F16 = 1, DKV_BF16 = 2 } dkv_dtype;

/* Bits of the device status word. */
#define DKV_DEV_BAD_SEQLEN   0x1   /* a sequence length outside [0, max_ctx] */
#define DKV_DEV_CAPACITY     0x2   /* an append would pass max_ctx (skipped) */
#define DKV_DEV_TIMEOUT      0x4   /* a bounded pipeline wait ran out */
#define DKV_DEV_BAD_HEADS    0x8   /* n_q_heads not a multiple of n_kv_heads */
#define DKV_DEV_BAD_PAGE     0x10  /* a block-table entry outside the page pool (skipped) */
#define DKV_DEV_BOUNDS       0x20  /* checked build only: a computed memory range outside its
                                      buffer (the access was skipped) */

typedef struct {
    int32_t batch;         /* B >= 1 (<= 1024) */
    int32_t n_kv_heads;    /* Hkv >= 1 */
    int32_t head_dim;      /* D, must be 128 */
    int32_t kf;            /* keyframe interval >= 1 (DKV_FMT_DELTA only) */
    int32_t max_ctx;       /* capacity in tokens per sequence, >= 1 */
    int32_t fmt;           /* dkv_format */
} dkv_cache_desc;

/* POD view of a cache laid out in caller-owned device memory.  Filled by
 * dkv_cache_init (contiguous) or dkv_cache_init_paged; all offsets are bytes
 * from `base`. */
typedef struct {
    dkv_cache_desc desc;
    void *base;
    size_t bytes;
    size_t seq_stride;     /* contiguous: bytes of one (batch, kv-head) sequence's data */
    size_t rec_bytes;      /* DELTA: bytes of one keyframe group record */
    int32_t n_groups;      /* DELTA: groups per sequence at capacity */
    int32_t reserved0;
    size_t off_data;       /* contiguous: compressed data, B*Hkv*seq_stride bytes */
    size_t off_state;      /* fp32 reconstruction state [2][B][Hkv][2][D] */
    size_t off_seqlen;     /* int32 seq_len[B] */
    size_t off_header;     /* int32 {status, counter, parity, reserved} */
    /* paged (DELTA only; page_groups == 0 for a contiguous cache): the records
     * live in a pool of pages; page i holds, for every kv head h, the records
     * of page_groups consecutive keyframe groups of one sequence, at
     * pool + i*page_bytes + (h*page_groups + g % page_groups)*rec_bytes, and
     * block_table[b*max_pages + g / page_groups] names the page of group g of
     * batch entry b. */
    void *pool;
    const int32_t *block_table;  /* device int32 [B][max_pages], caller-owned */
    size_t page_bytes;
    int64_t n_pages;
    int32_t page_groups;
    int32_t max_pages;
} dkv_cache;

/* ABI version of the loaded library (DKV_ABI_VERSION). */
int32_t dkv_abi_version(void);

/* Bytes of device memory a cache with this descriptor needs (0 if the
 * descriptor is invalid). */
size_t dkv_cache_bytes(const dkv_cache_desc *desc);

/* Lay a cache out in `dev` (>= dkv_cache_bytes, 256-byte aligned) and zero it
 * with cudaMemsetAsync on `stream` (every seq_len becomes 0).  Fills *out. */
dkv_status dkv_cache_init(const dkv_cache_desc *desc, void *dev, size_t bytes,
                          dkv_cache *out, void *stream);

/* Paged cache (a paged, group-aligned cache for ragged serving; the
 * "decoupled memory management" of page "DeltaKV ... Sparse-vLLM",
 * section "B. Sparse-vLLM", without the learned compressor).
 * dkv_cache_meta_bytes: bytes of the small metadata buffer a paged cache
 * needs (reconstruction state, lengths, header); dkv_page_bytes: bytes of one
 * page of page_groups keyframe groups (all kv heads), a multiple of 256.
 * Both return 0 for an invalid descriptor (or a format other than
 * DKV_FMT_DELTA, or page_groups < 1). */
size_t dkv_cache_meta_bytes(const dkv_cache_desc *desc);
size_t dkv_page_bytes(const dkv_cache_desc *desc, int32_t page_groups);

/* Lay out a paged cache: metadata in `meta` (>= dkv_cache_meta_bytes,
 * 256-byte aligned), records in `pool` (n_pages pages of dkv_page_bytes,
 * 256-byte aligned), pages named by `block_table` (device int32
 * [B][max_pages], 4-byte aligned, max_pages >= the pages max_ctx needs).
 * Zeroes the metadata and the pool with cudaMemsetAsync on `stream`.  The
 * block table stays caller-owned: entries may change between calls (a page
 * per page_groups*kf tokens of one sequence, never shared by two sequences);
 * a kernel that meets an entry outside [0, n_pages) sets DKV_DEV_BAD_PAGE and
 * skips that group.  DKV_FMT_DELTA only (DKV_EUNSUPPORTED otherwise).  Every
 * other call takes the resulting cache as it takes a contiguous one. */
dkv_status dkv_cache_init_paged(const dkv_cache_desc *desc, int32_t page_groups, void *pool,
                                int64_t n_pages, const int32_t *block_table, int32_t max_pages,
                                void *meta, size_t meta_bytes, dkv_cache *out, void *stream);

/* Encode whole sequences, replacing the cache contents.
 * K, V: [B][Hkv][T][D] contiguous device arrays of `dtype`.
 * seq_lens_dev: device int32[B] with 0 <= T_b <= T (NULL: every T_b = T).
 * Positions [0, T_b) of sequence b are encoded; seq_len[b] becomes T_b and
 * the reconstruction state is that of position T_b - 1.
 * (Format of the cache: keyframes, 4-bit closed-loop deltas, Q4_0 or fp16.) */
dkv_status dkv_encode(dkv_cache *cache, const void *K, const void *V, int32_t dtype,
                      const int32_t *seq_lens_dev, int32_t T, void *stream);

/* Append n_new tokens to every sequence at its current device-side seq_len,
 * continuing the closed loop from the stored reconstruction state.
 * K_new, V_new: [B][Hkv][n_new][D] contiguous device arrays of `dtype`.
 * A batch entry whose seq_len + n_new would pass max_ctx is skipped and sets
 * DKV_DEV_CAPACITY. */
dkv_status dkv_append(dkv_cache *cache, const void *K_new, const void *V_new,
                      int32_t dtype, int32_t n_new, void *stream);

/* Bytes of device workspace dkv_decode_attn needs for n_q_heads query heads on
 * the current device. */
size_t dkv_decode_workspace_bytes(const dkv_cache_desc *desc, int32_t n_q_heads);

/* One decode step of GQA attention over the cache: for every batch entry b
 * and query head h, out[b][h][:] = softmax(softmax_scale * q . k^_p) . v^_p
 * over the positions p < seq_len[b] (no mask beyond the length; an empty
 * sequence gives zeros).
 * Q: [B][n_q_heads][D] device array of q_dtype; out: [B][n_q_heads][D] fp32
 * device array; workspace: device scratch of >= dkv_decode_workspace_bytes;
 * softmax_scale must be finite and > 0 (DKV_EINVAL otherwise).  The kernels
 * multiply q as fp16 (fp32 queries as an fp16 hi + lo pair): fp16 and bf16
 * query values must lie within the fp16 range (|q| <= 65504; bf16 values
 * below 2^-14 keep an absolute error <= 2^-25).
 * Runs dkv_decode_attn_split then dkv_decode_attn_merge. */
dkv_status dkv_decode_attn(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                           int32_t n_q_heads, float softmax_scale, float *out,
                           void *workspace, size_t ws_bytes, void *stream);

/* The two launches of dkv_decode_attn, exposed so each can be timed alone:
 * the split kernel streams the compressed cache and writes per-range partial
 * (max, sum, unnormalised output) records to the workspace; the merge kernel
 * combines them (log-sum-exp) into out.  Same arguments as dkv_decode_attn. */
dkv_status dkv_decode_attn_split(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                                 int32_t n_q_heads, float softmax_scale,
                                 void *workspace, size_t ws_bytes, void *stream);
dkv_status dkv_decode_attn_merge(const dkv_cache *cache, int32_t n_q_heads, float *out,
                                 void *workspace, size_t ws_bytes, void *stream);

/* Multi-query decode (several new tokens per sequence, as in speculative
 * decoding).  The n_queries newest tokens of every sequence have
 * been appended (dkv_append with n_new = n_queries); query t (0 <= t <
 * n_queries) is token seq_len - n_queries + t's own query and attends to the
 * positions before seq_len - (n_queries - 1 - t), i.e. causally.
 * Q: [B][n_queries][n_q_heads][D] device array of q_dtype; out: the same
 * shape in fp32.  A query with no position gets zeros.  The queries of one kv
 * head are packed with its GQA heads into groups of 8 for the tensor cores
 * (n_queries * G <= 8 reads the cache once; each further group of 8 reads it
 * again).  1 <= n_queries <= 256; with n_queries = 1 this is dkv_decode_attn.
 * n_queries > 1 is for DKV_FMT_DELTA caches (DKV_EUNSUPPORTED otherwise).
 * Workspace: dkv_decode_workspace_bytes_mq. */
size_t dkv_decode_workspace_bytes_mq(const dkv_cache_desc *desc, int32_t n_q_heads,
                                     int32_t n_queries);
dkv_status dkv_decode_attn_mq(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                              int32_t n_q_heads, int32_t n_queries, float softmax_scale,
                              float *out, void *workspace, size_t ws_bytes, void *stream);

/* Fused append + decode (DKV_FMT_DELTA): the append of page "...Delta-KV",
 * section "핵심 아이디어", and the decode step of page "KV 캐시 벡터 양자화와
 * 주의 보존 변환", section "KV 캐시가 왜 병목인가", in one call.  The call
 * appends n_new tokens to every sequence, exactly as dkv_append would, and
 * runs the decode step
 * over the grown cache with the new tokens' own n_new queries, exactly as
 * dkv_decode_attn_mq with n_queries = n_new would (dkv_decode_attn for
 * n_new = 1).  The quantiser runs inside the decode's split kernel: the warps
 * that stream the groups the new tokens land in first quantise those tokens
 * (the same steps, in the same order, as the encoder: the stored codes, scales,
 * keyframes and reconstruction state are bit-identical to dkv_append's), so
 * the step takes two launches instead of three, and the merge publishes the
 * new lengths.
 * K_new, V_new: [B][Hkv][n_new][D] contiguous device arrays of kv_dtype (as
 * for dkv_append); Q: [B][n_new][n_q_heads][D] of q_dtype (for n_new = 1 that
 * is [B][n_q_heads][D]); out: the same shape as Q in fp32; workspace: >=
 * dkv_decode_workspace_bytes_mq(desc, n_q_heads, n_new).  A batch entry whose
 * tokens do not fit (seq_len + n_new > max_ctx) takes none, sets
 * DKV_DEV_CAPACITY and is decoded at its stored length; an invalid stored
 * length sets DKV_DEV_BAD_SEQLEN and decodes as empty.  1 <= n_new <= 256.
 * Other formats: DKV_EUNSUPPORTED.  A bad block-table entry (paged cache) sets
 * DKV_DEV_BAD_PAGE; the tokens of that page are then not stored.
 * The _split and _merge halves are the two launches, exposed so each can be
 * timed alone; they must run back to back on one stream with the same
 * arguments, with no other call on the cache between them. */
dkv_status dkv_append_decode_attn(dkv_cache *cache, const void *K_new, const void *V_new,
                                  int32_t kv_dtype, int32_t n_new, const void *Q,
                                  int32_t q_dtype, int32_t n_q_heads, float softmax_scale,
                                  float *out, void *workspace, size_t ws_bytes, void *stream);
dkv_status dkv_append_decode_attn_split(dkv_cache *cache, const void *K_new, const void *V_new,
                                        int32_t kv_dtype, int32_t n_new, const void *Q,
                                        int32_t q_dtype, int32_t n_q_heads, float softmax_scale,
                                        void *workspace, size_t ws_bytes, void *stream);
dkv_status dkv_append_decode_attn_merge(dkv_cache *cache, int32_t n_new, int32_t n_q_heads,
                                        float *out, void *workspace, size_t ws_bytes,
                                        void *stream);

/* Long-range reference encoding: the training-free part of DeltaKV (page
 * "DeltaKV" summary, section 2: similar tokens lie far apart in the context;
 * section A: "Strided Reference Selection", "Residual Encoding",
 * "Reconstruction"; section 4, "양자화 친화성": the residuals take 4-bit
 * quantisation), with the learned compressor replaced by the Q4_0 block rule.
 * Every stride-th token (p mod stride == 0) is a reference, stored as fp16.
 * Every other token p takes the n_refs references r < p nearest to it
 * (squared Euclidean distance to the stored reference, binary64, channels in
 * order; ties to the smaller position; all of them when fewer exist), and
 * stores its residual against their mean (binary32 sum in ascending position
 * divided by their count) with the Q4_0 block rule; x^ = mean + (code - 8) d.
 * n_seq independent sequences.  X: [n_seq][T][128] device array of dtype.
 * Outputs (device, caller-owned, canonical layouts):
 *   ref        int32  [n_seq][T][n_refs]   chosen reference numbers r / stride,
 *                                          ascending; -1 unused / reference rows
 *   ref_values uint16 [n_seq][ceil(T/stride)][128]  fp16 bits of the references
 *   scales     uint16 [n_seq][T][4]         fp16 bits (0 on reference rows)
 *   codes      uint8  [n_seq][T][128]       0..15 (0 on reference rows)
 *   xhat       float  [n_seq][T][128]       reconstruction (NULL: not written)
 * 1 <= n_refs <= 8, stride >= 1.  dkv_lr_decode_attn attends over these
 * outputs. */
dkv_status dkv_lr_encode(const void *X, int32_t dtype, int32_t n_seq, int32_t T, int32_t stride,
                         int32_t n_refs, int32_t *ref, uint16_t *ref_values, uint16_t *scales,
                         uint8_t *codes, float *xhat, void *stream);

/* One tensor (K or V) of a long-range reference encoding, in the canonical
 * layouts dkv_lr_encode writes (device arrays, 16-byte aligned, caller-owned);
 * sequence index = batch entry * n_kv_heads + kv head. */
typedef struct {
    const int32_t *ref;          /* [n_seq][T][n_refs] */
    const uint16_t *ref_values;  /* [n_seq][ceil(T/stride)][128] */
    const uint16_t *scales;      /* [n_seq][T][4] */
    const uint8_t *codes;        /* [n_seq][T][128] */
} dkv_lr_tensor;

/* Decode attention over the long-range reference encoding (page "DeltaKV"
 * summary, section A, "Reconstruction": the residual plus the mean of the
 * chosen references; the decode step of page "KV 캐시 벡터 양자화와 주의 보존
 * 변환", section "KV 캐시가 왜 병목인가").  For batch entry b and query head h
 * (kv head h / (n_q_heads / n_kv_heads)): out[b][h] = softmax over p < len_b
 * of softmax_scale * q . k^_p, applied to v^_p, where x^ is the encoding's
 * reconstruction (a reference token: its fp16 value; any other token: the
 * mean of its references plus its dequantised residual).  The reconstruction
 * is never formed: the scores are the mean of the references' dot products
 * plus q . residual, and the output is sum_r W_r v^_r plus the residuals
 * weighted by the softmax (W_r: the weight each reference receives from the
 * tokens that use it).  K and V are encoded separately (each with its own
 * choices), with the same T, stride and n_refs.
 * lens_dev: device int32[batch], 0 <= len_b <= T (NULL: every len_b = T); a
 * sequence of length 0 gives zeros.  Q: [batch][n_q_heads][128] of q_dtype
 * (fp32 queries are split into an fp16 hi + lo pair); out: the same shape,
 * fp32.  n_q_heads / n_kv_heads must be 1..8 (DKV_EUNSUPPORTED otherwise);
 * softmax_scale finite and > 0.  workspace: >= dkv_lr_decode_workspace_bytes.
 * Three launches on `stream`: the references' dot products, one warp per
 * 256-token chunk (scores, softmax, residual part), one block per sequence
 * (combine and reference part). */
size_t dkv_lr_decode_workspace_bytes(int32_t batch, int32_t n_kv_heads, int32_t T,
                                     int32_t stride);
dkv_status dkv_lr_decode_attn(const dkv_lr_tensor *K, const dkv_lr_tensor *V, int32_t batch,
                              int32_t n_kv_heads, int32_t T, int32_t stride, int32_t n_refs,
                              const int32_t *lens_dev, const void *Q, int32_t q_dtype,
                              int32_t n_q_heads, float softmax_scale, float *out,
                              void *workspace, size_t ws_bytes, void *stream);

/* Size of the library-owned scratch array used by dkv_decode_attn_noalloc. */
#define DKV_NOALLOC_SCRATCH_BYTES (16u << 20)

/* dkv_decode_attn for callers that cannot allocate device memory when they
 * decode (for example code running under CUDA graph capture, where cudaMalloc
 * is not allowed, or a plugin inside an engine that owns and pre-plans every
 * device allocation).  The pages have no counterpart: this is a deployment
 * variant of the same decode step, with the same arguments minus the
 * workspace.  The partial records go to a fixed 16 MiB array that the library
 * itself holds on every GPU that loads it, until the process exits.  The
 * first call on a device looks up that array's address (make it before any
 * stream capture); the lookup is repeated only when the device's context has
 * changed since (cudaDeviceReset loads the library's device code anew, so
 * the array may move), which again must not happen under capture.  The cache
 * is validated first, with the statuses of dkv_decode_attn (DKV_EINVAL,
 * DKV_EALIGN, DKV_EUNSUPPORTED); then DKV_ECAPACITY when the step needs more
 * than DKV_NOALLOC_SCRATCH_BYTES of records (see dkv_decode_workspace_bytes);
 * DKV_ECUDA only for a failed device query or launch.  All calls share the
 * array: calls that overlap on the GPU race and must be serialised by the
 * caller.  Allocates and frees nothing. */
dkv_status dkv_decode_attn_noalloc(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                                   int32_t n_q_heads, float softmax_scale, float *out,
                                   void *stream);

/* Copy the stored fields out in a canonical, layout-independent form (device
 * destinations; NULL skips a field):
 *   codes     uint8  [B][Hkv][2][max_ctx][D]   one code per element
 *   scales    uint16 [B][Hkv][2][max_ctx][D/32] fp16 bits of the block scale
 *   keyframes uint16 [B][Hkv][2][n_kf][D]     fp16 bits; n_kf = n_groups
 *                                             (DELTA) or max_ctx (FP16)
 *   state     float  [B][Hkv][2][D]           reconstruction of the last
 *                                             encoded position (DELTA)
 * Rows of keyframe positions in codes/scales are zero (DELTA).  Tensor index
 * 0 is K, 1 is V. */
dkv_status dkv_export_canonical(const dkv_cache *cache, uint8_t *codes, uint16_t *scales,
                                uint16_t *keyframes, float *state, void *stream);

/* Reconstructed values x^ of every stored position, fp32
 * [B][Hkv][2][max_ctx][D] (positions >= seq_len are left untouched). */
dkv_status dkv_dequantize(const dkv_cache *cache, float *out, void *stream);

/* Synchronise `stream`, copy the device status word to *host_out and clear
 * it.  Returns DKV_EDEVICE if it was non-zero, DKV_OK otherwise. */
dkv_status dkv_get_device_status(const dkv_cache *cache, int32_t *host_out, void *stream);

/* Test support for failure detection (no counterpart on the pages).  With
 * mode 1, later decode-attention split launches from this process arm their
 * copy barriers without issuing the copies, so every bounded pipeline wait
 * runs out (after about a second) and the kernel records DKV_DEV_TIMEOUT in
 * the status word and returns, instead of hanging; the outputs of such a
 * launch are meaningless.  With mode 2, those launches are told the workspace
 * is two partial records smaller than it is: the bounds-checked build
 * (DKV_CHECKED) then records DKV_DEV_BOUNDS and skips the last record's
 * writes (the buffer itself is large enough, so nothing is touched out of
 * range); other builds ignore it.  Mode 0 restores normal operation.  Nothing
 * traps or faults either way.  Not thread-safe; meant for tests. */
void dkv_debug_set_fault(int32_t mode);

/* Test support (no counterpart on the pages): checks the quotient the
 * delta encoder uses (one correctly rounded reciprocal of the block scale,
 * then Markstein's exact-residual correction) against the IEEE division
 * __fdiv_rn, for every finite non-zero fp16 divisor b and, for each of the n
 * multipliers u_dev[i] (device fp32, 16-byte aligned), the dividends
 * a = RN(u_i b) and its two floating-point neighbours.  Adds to
 * *mismatches_dev (device uint64, 16-byte aligned; the caller zeroes it) the
 * number of cases where the two quotients differ in a bit while the IEEE
 * quotient is a normal number, or give different codes trunc(q + 8.5)
 * clamped to 0..15 (a quotient below the normal range -- possible only when
 * a itself is subnormal -- always gives code 8, so its last bit is free).
 * Asynchronous on `stream`. */
dkv_status dkv_debug_division_check(const float *u_dev, int32_t n, uint64_t *mismatches_dev,
                                    void *stream);

/* Static description of a status code. */
const char *dkv_status_str(dkv_status s);

#ifdef __cplusplus
}
#endif
#endif /* DKV_H */
