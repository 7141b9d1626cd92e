// dkv_api.cu -- the C ABI (include/dkv.h): argument validation, cache layout,
// and the launches.  Nothing here allocates device memory; every launch goes
// on the caller's stream.
#include <cstdint>
#include <cstring>
#include <initializer_list>

#include "../../include/dkv.h"
#include "dkv_common.cuh"
#include "dkv_internal.h"

namespace {

using dkv::CacheView;

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct Layout {
    size_t seq_stride, rec_bytes, off_data, off_state, off_seqlen, off_header, total;
    int32_t n_groups;
};

dkv_status check_desc(const dkv_cache_desc *d) {
    if (!d) return DKV_EINVAL;
    if (d->fmt != DKV_FMT_FP16 && d->fmt != DKV_FMT_Q4_0 && d->fmt != DKV_FMT_DELTA)
        return DKV_EINVAL;
    if (d->batch < 1 || d->batch > 1024 || d->n_kv_heads < 1 || d->n_kv_heads > 4096)
        return DKV_EINVAL;
    if (d->max_ctx < 1 || d->max_ctx > (1 << 28)) return DKV_EINVAL;
    if (d->fmt == DKV_FMT_DELTA && (d->kf < 1 || d->kf > (1 << 20))) return DKV_EINVAL;
    if (d->head_dim != dkv::D) return DKV_EUNSUPPORTED;
    return DKV_OK;
}

// paged: no data area (the records live in the page pool); the metadata
// starts at the buffer's beginning
Layout make_layout(const dkv_cache_desc *d, bool paged = false) {
    Layout L{};
    const size_t cap = (size_t)d->max_ctx;
    if (d->fmt == DKV_FMT_DELTA) {
        L.rec_bytes = (size_t)dkv::delta_rec_bytes(d->kf);
        L.n_groups = (int32_t)((cap + d->kf - 1) / d->kf);
        L.seq_stride = L.rec_bytes * (size_t)L.n_groups;
    } else if (d->fmt == DKV_FMT_Q4_0) {
        L.rec_bytes = 0;
        L.n_groups = 0;
        L.seq_stride = cap * dkv::POS_Q4;
    } else {
        L.rec_bytes = 0;
        L.n_groups = 0;
        L.seq_stride = cap * dkv::POS_F16;
    }
    const size_t nseq = (size_t)d->batch * d->n_kv_heads;
    L.off_data = 0;
    L.off_state = paged ? 0 : align_up(nseq * L.seq_stride + 4096, kAlign);
    L.off_seqlen = align_up(L.off_state + 2 * nseq * 2 * dkv::D * sizeof(float), kAlign);
    L.off_header = align_up(L.off_seqlen + (size_t)d->batch * sizeof(int32_t), kAlign);
    L.total = align_up(L.off_header + 16, kAlign);
    return L;
}

size_t page_bytes_of(const dkv_cache_desc *d, int32_t pg) {
    return align_up((size_t)d->n_kv_heads * (size_t)pg * (size_t)dkv::delta_rec_bytes(d->kf),
                    kAlign);
}

dkv_status check_cache(const dkv_cache *c) {
    if (!c || !c->base) return DKV_EINVAL;
    dkv_status s = check_desc(&c->desc);
    if (s != DKV_OK) return s;
    const bool paged = c->page_groups != 0;
    Layout L = make_layout(&c->desc, paged);
    if (c->bytes < L.total || c->seq_stride != L.seq_stride || c->off_header != L.off_header)
        return DKV_EINVAL;
    if ((reinterpret_cast<uintptr_t>(c->base) & (kAlign - 1)) != 0) return DKV_EALIGN;
    if (paged) {
        if (c->desc.fmt != DKV_FMT_DELTA || c->page_groups < 1 || !c->pool || !c->block_table ||
            c->n_pages < 1 || c->page_bytes != page_bytes_of(&c->desc, c->page_groups) ||
            (int64_t)c->max_pages * c->page_groups < L.n_groups)
            return DKV_EINVAL;
        if ((reinterpret_cast<uintptr_t>(c->pool) & (kAlign - 1)) != 0 ||
            (reinterpret_cast<uintptr_t>(c->block_table) & 3) != 0)
            return DKV_EALIGN;
    }
    return DKV_OK;
}

CacheView view_of(const dkv_cache *c) {
    CacheView v;
    uint8_t *base = static_cast<uint8_t *>(c->base);
    v.data = base + c->off_data;
    v.data_bytes = (int64_t)c->desc.batch * c->desc.n_kv_heads * (int64_t)c->seq_stride;
    v.state = reinterpret_cast<float *>(base + c->off_state);
    v.seqlen = reinterpret_cast<int32_t *>(base + c->off_seqlen);
    v.header = reinterpret_cast<int32_t *>(base + c->off_header);
    v.seq_stride = (int64_t)c->seq_stride;
    v.rec_bytes = (int64_t)c->rec_bytes;
    v.B = c->desc.batch;
    v.Hkv = c->desc.n_kv_heads;
    v.kf = c->desc.fmt == DKV_FMT_DELTA ? c->desc.kf : 1;
    v.pool = static_cast<uint8_t *>(c->pool);
    v.bt = c->block_table;
    v.page_bytes = (int64_t)c->page_bytes;
    v.n_pages = c->n_pages;
    v.pg = c->page_groups;
    v.maxp = c->max_pages;
    v.cap = c->desc.max_ctx;
    v.fmt = c->desc.fmt;
    v.n_groups = c->n_groups;
    v.len_add = 0;
    return v;
}

inline dkv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DKV_OK : DKV_ECUDA; }

int g_debug_fault = 0;   // dkv_debug_set_fault

inline bool valid_dtype(int32_t t) { return t == DKV_F32 || t == DKV_F16 || t == DKV_BF16; }

constexpr int32_t kMaxQueries = 256;

int64_t workspace_floats(const dkv_cache_desc *d, int32_t Hq, int32_t nq, bool *ok) {
    *ok = false;
    if (check_desc(d) != DKV_OK || Hq < 1 || Hq % d->n_kv_heads != 0) return 0;
    if (nq < 1 || nq > kMaxQueries) return 0;
    const int G = Hq / d->n_kv_heads;
    const int64_t nhg = ((int64_t)nq * G + 7) / 8;
    dkv::SplitGeom g;
    if (dkv::split_geometry(d->fmt, d->kf,
                            dkv::split_max_units(d->fmt, d->kf, d->batch, d->n_kv_heads, (int)nhg,
                                                 d->max_ctx),
                            &g) != cudaSuccess)
        return 0;
    const int64_t NW = (int64_t)g.ctas * g.warps_per_cta;
    const int64_t slots = NW + (int64_t)d->batch * d->n_kv_heads * nhg;
    *ok = true;
    // + the decoded lengths of a fused append + decode, int32[B]
    int64_t f = slots * dkv::PARTIAL_FLOATS + ((int64_t)d->batch + 3) / 4 * 4;
    // kf > 32: + per warp, a record of the group its range enters midway and
    // the state it hands on
    if (d->fmt == DKV_FMT_DELTA && d->kf > 32)
        f += NW * (dkv::PARTIAL_FLOATS + dkv::HANDOFF_FLOATS) + dkv::HAND_HDR;
    return f;
}

dkv_status check_decode(const dkv_cache *cache, const void *Q, int32_t q_dtype, int32_t Hq,
                        int32_t nq, void *ws, size_t ws_bytes, int64_t *need_floats) {
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (!ws || (Q == nullptr && q_dtype >= 0)) return DKV_EINVAL;
    if (q_dtype >= 0 && !valid_dtype(q_dtype)) return DKV_EINVAL;
    if (Hq < 1 || Hq % cache->desc.n_kv_heads != 0) return DKV_EINVAL;
    if (nq < 1 || nq > kMaxQueries) return DKV_EINVAL;
    if ((Q && !aligned16(Q)) || !aligned16(ws)) return DKV_EALIGN;
    bool ok;
    int64_t need = workspace_floats(&cache->desc, Hq, nq, &ok);
    if (!ok) return DKV_ECUDA;
    if (ws_bytes < (size_t)need * sizeof(float)) return DKV_ECAPACITY;
    *need_floats = need;
    return DKV_OK;
}

}  // namespace

dkv_status dkv::validate_cache(const dkv_cache *c) { return check_cache(c); }

extern "C" {

int32_t dkv_abi_version(void) { return DKV_ABI_VERSION; }

size_t dkv_cache_bytes(const dkv_cache_desc *desc) {
    if (check_desc(desc) != DKV_OK) return 0;
    return make_layout(desc).total;
}

dkv_status dkv_cache_init(const dkv_cache_desc *desc, void *dev, size_t bytes, dkv_cache *out,
                          void *stream) {
    dkv_status s = check_desc(desc);
    if (s != DKV_OK) return s;
    if (!dev || !out) return DKV_EINVAL;
    if ((reinterpret_cast<uintptr_t>(dev) & (kAlign - 1)) != 0) return DKV_EALIGN;
    Layout L = make_layout(desc);
    if (bytes < L.total) return DKV_ECAPACITY;
    std::memset(out, 0, sizeof(*out));
    out->desc = *desc;
    out->base = dev;
    out->bytes = bytes;
    out->seq_stride = L.seq_stride;
    out->rec_bytes = L.rec_bytes;
    out->n_groups = L.n_groups;
    out->off_data = L.off_data;
    out->off_state = L.off_state;
    out->off_seqlen = L.off_seqlen;
    out->off_header = L.off_header;
    return cuda_status(cudaMemsetAsync(dev, 0, L.total, static_cast<cudaStream_t>(stream)));
}

size_t dkv_cache_meta_bytes(const dkv_cache_desc *desc) {
    if (check_desc(desc) != DKV_OK || desc->fmt != DKV_FMT_DELTA) return 0;
    return make_layout(desc, true).total;
}

size_t dkv_page_bytes(const dkv_cache_desc *desc, int32_t page_groups) {
    if (check_desc(desc) != DKV_OK || desc->fmt != DKV_FMT_DELTA || page_groups < 1) return 0;
    return page_bytes_of(desc, page_groups);
}

dkv_status dkv_cache_init_paged(const dkv_cache_desc *desc, int32_t page_groups, void *pool,
                                int64_t n_pages, const int32_t *block_table, int32_t max_pages,
                                void *meta, size_t meta_bytes, dkv_cache *out, void *stream) {
    dkv_status s = check_desc(desc);
    if (s != DKV_OK) return s;
    if (desc->fmt != DKV_FMT_DELTA) return DKV_EUNSUPPORTED;
    if (!pool || !block_table || !meta || !out || page_groups < 1 || n_pages < 1 ||
        max_pages < 1)
        return DKV_EINVAL;
    if ((reinterpret_cast<uintptr_t>(pool) & (kAlign - 1)) != 0 ||
        (reinterpret_cast<uintptr_t>(meta) & (kAlign - 1)) != 0 ||
        (reinterpret_cast<uintptr_t>(block_table) & 3) != 0)
        return DKV_EALIGN;
    Layout L = make_layout(desc, true);
    if ((int64_t)max_pages * page_groups < L.n_groups) return DKV_EINVAL;
    if (meta_bytes < L.total) return DKV_ECAPACITY;
    std::memset(out, 0, sizeof(*out));
    out->desc = *desc;
    out->base = meta;
    out->bytes = meta_bytes;
    out->seq_stride = L.seq_stride;
    out->rec_bytes = L.rec_bytes;
    out->n_groups = L.n_groups;
    out->off_data = 0;
    out->off_state = L.off_state;
    out->off_seqlen = L.off_seqlen;
    out->off_header = L.off_header;
    out->pool = pool;
    out->block_table = block_table;
    out->page_bytes = page_bytes_of(desc, page_groups);
    out->n_pages = n_pages;
    out->page_groups = page_groups;
    out->max_pages = max_pages;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(meta, 0, L.total, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(pool, 0, (size_t)n_pages * out->page_bytes, st);
    return cuda_status(e);
}

dkv_status dkv_encode(dkv_cache *cache, const void *K, const void *V, int32_t dtype,
                      const int32_t *seq_lens_dev, int32_t T, void *stream) {
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (!K || !V || !valid_dtype(dtype) || T < 1) return DKV_EINVAL;
    if (!aligned16(K) || !aligned16(V) || (seq_lens_dev && !aligned16(seq_lens_dev)))
        return DKV_EALIGN;
    if (T > cache->desc.max_ctx) return DKV_ECAPACITY;
    CacheView v = view_of(cache);
    return cuda_status(dkv::launch_encode(v, K, V, dtype, seq_lens_dev, T, 0,
                                          static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_append(dkv_cache *cache, const void *K_new, const void *V_new, int32_t dtype,
                      int32_t n_new, void *stream) {
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (!K_new || !V_new || !valid_dtype(dtype) || n_new < 1) return DKV_EINVAL;
    if (!aligned16(K_new) || !aligned16(V_new)) return DKV_EALIGN;
    if (n_new > cache->desc.max_ctx) return DKV_ECAPACITY;
    CacheView v = view_of(cache);
    return cuda_status(dkv::launch_encode(v, K_new, V_new, dtype, nullptr, n_new, 1,
                                          static_cast<cudaStream_t>(stream)));
}

size_t dkv_decode_workspace_bytes(const dkv_cache_desc *desc, int32_t n_q_heads) {
    return dkv_decode_workspace_bytes_mq(desc, n_q_heads, 1);
}

size_t dkv_decode_workspace_bytes_mq(const dkv_cache_desc *desc, int32_t n_q_heads,
                                     int32_t n_queries) {
    bool ok;
    int64_t f = workspace_floats(desc, n_q_heads, n_queries, &ok);
    return ok ? (size_t)f * sizeof(float) : 0;
}

dkv_status dkv_decode_attn_split(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                                 int32_t n_q_heads, float softmax_scale, void *workspace,
                                 size_t ws_bytes, void *stream) {
    int64_t need;
    if (!Q) return DKV_EINVAL;
    if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return DKV_EINVAL;  // finite, > 0
    dkv_status s = check_decode(cache, Q, q_dtype, n_q_heads, 1, workspace, ws_bytes, &need);
    if (s != DKV_OK) return s;
    CacheView v = view_of(cache);
    return cuda_status(dkv::launch_split(v, Q, q_dtype, n_q_heads, 1, softmax_scale,
                                         static_cast<float *>(workspace), need, g_debug_fault,
                                         static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_decode_attn_merge(const dkv_cache *cache, int32_t n_q_heads, float *out,
                                 void *workspace, size_t ws_bytes, void *stream) {
    int64_t need;
    if (!out) return DKV_EINVAL;
    dkv_status s = check_decode(cache, nullptr, -1, n_q_heads, 1, workspace, ws_bytes, &need);
    if (s != DKV_OK) return s;
    if (!aligned16(out)) return DKV_EALIGN;
    CacheView v = view_of(cache);
    return cuda_status(dkv::launch_merge(v, n_q_heads, 1, out, static_cast<const float *>(workspace),
                                         need, static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_decode_attn(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                           int32_t n_q_heads, float softmax_scale, float *out, void *workspace,
                           size_t ws_bytes, void *stream) {
    if (!out) return DKV_EINVAL;
    if (!aligned16(out)) return DKV_EALIGN;
    dkv_status s = dkv_decode_attn_split(cache, Q, q_dtype, n_q_heads, softmax_scale, workspace,
                                         ws_bytes, stream);
    if (s != DKV_OK) return s;
    return dkv_decode_attn_merge(cache, n_q_heads, out, workspace, ws_bytes, stream);
}

dkv_status dkv_decode_attn_mq(const dkv_cache *cache, const void *Q, int32_t q_dtype,
                              int32_t n_q_heads, int32_t n_queries, float softmax_scale,
                              float *out, void *workspace, size_t ws_bytes, void *stream) {
    if (!out || !Q) return DKV_EINVAL;
    if (!aligned16(out)) return DKV_EALIGN;
    if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return DKV_EINVAL;  // finite, > 0
    int64_t need;
    dkv_status s = check_decode(cache, Q, q_dtype, n_q_heads, n_queries, workspace, ws_bytes,
                                &need);
    if (s != DKV_OK) return s;
    if (n_queries > 1 && cache->desc.fmt != DKV_FMT_DELTA) return DKV_EUNSUPPORTED;
    CacheView v = view_of(cache);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *ws = static_cast<float *>(workspace);
    cudaError_t e = dkv::launch_split(v, Q, q_dtype, n_q_heads, n_queries, softmax_scale, ws,
                                      need, g_debug_fault, st);
    if (e == cudaSuccess) e = dkv::launch_merge(v, n_q_heads, n_queries, out, ws, need, st);
    return cuda_status(e);
}

dkv_status dkv_append_decode_attn_split(dkv_cache *cache, const void *K_new, const void *V_new,
                                        int32_t kv_dtype, int32_t n_new, const void *Q,
                                        int32_t q_dtype, int32_t n_q_heads, float softmax_scale,
                                        void *workspace, size_t ws_bytes, void *stream) {
    if (!Q || !K_new || !V_new || !valid_dtype(kv_dtype)) return DKV_EINVAL;
    if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return DKV_EINVAL;  // finite, > 0
    if (!aligned16(K_new) || !aligned16(V_new)) return DKV_EALIGN;
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (cache->desc.fmt != DKV_FMT_DELTA) return DKV_EUNSUPPORTED;
    int64_t need;
    s = check_decode(cache, Q, q_dtype, n_q_heads, n_new, workspace, ws_bytes, &need);
    if (s != DKV_OK) return s;
    if (n_new > cache->desc.max_ctx) return DKV_ECAPACITY;
    CacheView v = view_of(cache);
    v.len_add = n_new;
    return cuda_status(dkv::launch_split(v, Q, q_dtype, n_q_heads, n_new, softmax_scale,
                                         static_cast<float *>(workspace), need, g_debug_fault,
                                         static_cast<cudaStream_t>(stream), K_new, V_new,
                                         kv_dtype));
}

dkv_status dkv_append_decode_attn_merge(dkv_cache *cache, int32_t n_new, int32_t n_q_heads,
                                        float *out, void *workspace, size_t ws_bytes,
                                        void *stream) {
    if (!out) return DKV_EINVAL;
    if (!aligned16(out)) return DKV_EALIGN;
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (cache->desc.fmt != DKV_FMT_DELTA) return DKV_EUNSUPPORTED;
    int64_t need;
    s = check_decode(cache, nullptr, -1, n_q_heads, n_new, workspace, ws_bytes, &need);
    if (s != DKV_OK) return s;
    if (n_new > cache->desc.max_ctx) return DKV_ECAPACITY;
    CacheView v = view_of(cache);
    v.len_add = n_new;
    return cuda_status(dkv::launch_merge(v, n_q_heads, n_new, out,
                                         static_cast<const float *>(workspace), need,
                                         static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_append_decode_attn(dkv_cache *cache, const void *K_new, const void *V_new,
                                  int32_t kv_dtype, int32_t n_new, const void *Q,
                                  int32_t q_dtype, int32_t n_q_heads, float softmax_scale,
                                  float *out, void *workspace, size_t ws_bytes, void *stream) {
    if (!out) return DKV_EINVAL;
    if (!aligned16(out)) return DKV_EALIGN;
    dkv_status s = dkv_append_decode_attn_split(cache, K_new, V_new, kv_dtype, n_new, Q, q_dtype,
                                                n_q_heads, softmax_scale, workspace, ws_bytes,
                                                stream);
    if (s != DKV_OK) return s;
    return dkv_append_decode_attn_merge(cache, n_new, n_q_heads, out, workspace, ws_bytes, stream);
}

dkv_status dkv_lr_encode(const void *X, int32_t dtype, int32_t n_seq, int32_t T, int32_t stride,
                         int32_t n_refs, int32_t *ref, uint16_t *ref_values, uint16_t *scales,
                         uint8_t *codes, float *xhat, void *stream) {
    if (!X || !ref || !ref_values || !scales || !codes || !valid_dtype(dtype)) return DKV_EINVAL;
    if (n_seq < 1 || n_seq > 65535 || T < 1 || stride < 1 || n_refs < 1 || n_refs > 8)
        return DKV_EINVAL;
    if ((int64_t)n_seq * T > ((int64_t)1 << 31)) return DKV_ECAPACITY;
    if (!aligned16(X) || !aligned16(ref) || !aligned16(ref_values) || !aligned16(scales) ||
        !aligned16(codes) || (xhat && !aligned16(xhat)))
        return DKV_EALIGN;
    return cuda_status(dkv::launch_lr_encode(X, dtype, n_seq, T, stride, n_refs, ref, ref_values,
                                             scales, codes, xhat,
                                             static_cast<cudaStream_t>(stream)));
}

size_t dkv_lr_decode_workspace_bytes(int32_t batch, int32_t n_kv_heads, int32_t T,
                                     int32_t stride) {
    if (batch < 1 || n_kv_heads < 1 || T < 1 || stride < 1) return 0;
    if ((int64_t)batch * n_kv_heads * T > ((int64_t)1 << 31)) return 0;
    return dkv::lrd_workspace_floats(batch, n_kv_heads, T, stride) * sizeof(float);
}

dkv_status dkv_lr_decode_attn(const dkv_lr_tensor *K, const dkv_lr_tensor *V, int32_t batch,
                              int32_t n_kv_heads, int32_t T, int32_t stride, int32_t n_refs,
                              const int32_t *lens_dev, const void *Q, int32_t q_dtype,
                              int32_t n_q_heads, float softmax_scale, float *out,
                              void *workspace, size_t ws_bytes, void *stream) {
    if (!K || !V || !Q || !out || !workspace || !valid_dtype(q_dtype)) return DKV_EINVAL;
    for (const dkv_lr_tensor *t : {K, V}) {
        if (!t->ref || !t->ref_values || !t->scales || !t->codes) return DKV_EINVAL;
        if (!aligned16(t->ref) || !aligned16(t->ref_values) || !aligned16(t->scales) ||
            !aligned16(t->codes))
            return DKV_EALIGN;
    }
    if (batch < 1 || batch > 65535 || n_kv_heads < 1 || T < 1 || stride < 1 || n_refs < 1 ||
        n_refs > 8 || n_q_heads < 1 || n_q_heads % n_kv_heads != 0)
        return DKV_EINVAL;
    if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return DKV_EINVAL;
    if (n_q_heads / n_kv_heads > 8) return DKV_EUNSUPPORTED;
    if (!aligned16(Q) || !aligned16(out) || !aligned16(workspace) ||
        (lens_dev && (reinterpret_cast<uintptr_t>(lens_dev) & 3)))
        return DKV_EALIGN;
    const size_t need = dkv_lr_decode_workspace_bytes(batch, n_kv_heads, T, stride);
    if (need == 0) return DKV_ECAPACITY;
    if (ws_bytes < need) return DKV_ECAPACITY;
    const dkv::LrdView kv{K->ref, K->ref_values, K->scales, K->codes};
    const dkv::LrdView vv{V->ref, V->ref_values, V->scales, V->codes};
    return cuda_status(dkv::launch_lr_decode(kv, vv, batch, n_kv_heads, T, stride, n_refs,
                                             lens_dev, Q, q_dtype, n_q_heads, softmax_scale, out,
                                             static_cast<float *>(workspace),
                                             static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_export_canonical(const dkv_cache *cache, uint8_t *codes, uint16_t *scales,
                                uint16_t *keyframes, float *state, void *stream) {
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if ((codes && !aligned16(codes)) || (scales && !aligned16(scales)) ||
        (keyframes && !aligned16(keyframes)) || (state && !aligned16(state)))
        return DKV_EALIGN;
    CacheView v = view_of(cache);
    return cuda_status(dkv::launch_readback(v, codes, scales, keyframes, state, nullptr,
                                            static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_dequantize(const dkv_cache *cache, float *out, void *stream) {
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (!out) return DKV_EINVAL;
    if (!aligned16(out)) return DKV_EALIGN;
    CacheView v = view_of(cache);
    return cuda_status(dkv::launch_readback(v, nullptr, nullptr, nullptr, nullptr, out,
                                            static_cast<cudaStream_t>(stream)));
}

dkv_status dkv_get_device_status(const dkv_cache *cache, int32_t *host_out, void *stream) {
    dkv_status s = check_cache(cache);
    if (s != DKV_OK) return s;
    if (!host_out) return DKV_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t *word = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(cache->base) + cache->off_header);
    int32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, word, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return DKV_ECUDA;
    *host_out = h;
    return h ? DKV_EDEVICE : DKV_OK;
}

void dkv_debug_set_fault(int32_t mode) { g_debug_fault = (mode == 1 || mode == 2) ? mode : 0; }

dkv_status dkv_debug_division_check(const float *u_dev, int32_t n, uint64_t *mismatches_dev,
                                    void *stream) {
    if (!u_dev || !mismatches_dev || n < 1) return DKV_EINVAL;
    if (!aligned16(u_dev) || !aligned16(mismatches_dev)) return DKV_EALIGN;
    return cuda_status(dkv::launch_division_check(
        u_dev, n, reinterpret_cast<unsigned long long *>(mismatches_dev),
        static_cast<cudaStream_t>(stream)));
}

const char *dkv_status_str(dkv_status s) {
    switch (s) {
        case DKV_OK: return "ok";
        case DKV_EINVAL: return "invalid argument";
        case DKV_EALIGN: return "misaligned pointer";
        case DKV_ECAPACITY: return "capacity or workspace too small";
        case DKV_EUNSUPPORTED: return "unsupported configuration";
        case DKV_ECUDA: return "CUDA error";
        case DKV_EDEVICE: return "device status word set";
    }
    return "unknown status";
}

}  // extern "C"
