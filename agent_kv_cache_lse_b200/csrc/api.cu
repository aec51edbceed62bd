// C-ABI entry points of libkvc: argument validation, geometry, dispatch to the
// kernels, error strings.  Every step of the path runs in CUDA kernels; this file
// only checks arguments and enqueues launches.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/kvc.h"
#include "internal.h"

namespace {

thread_local char g_err[512] = "";

kvc_status fail(kvc_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

kvc_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return KVC_OK;
    return fail(KVC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int64_t kMaxRows = 65534;

kvc_status view_cache(const kvc_cache *c, kvc::CacheView &v, bool need_pools) {
    if (!c) return fail(KVC_ERR_INVALID_ARGUMENT, "cache is NULL");
    if (c->num_seqs <= 0 || c->num_layers <= 0 || c->num_kv_heads <= 0)
        return fail(KVC_ERR_INVALID_ARGUMENT, "num_seqs, num_layers and num_kv_heads must be positive");
    const int64_t rows = (int64_t)c->num_seqs * c->num_layers * c->num_kv_heads;
    if (rows > kMaxRows) return fail(KVC_ERR_UNSUPPORTED, "at most %lld rows per call", (long long)kMaxRows);
    if (c->page_size <= 0 || c->page_size > 4096) return fail(KVC_ERR_INVALID_ARGUMENT, "page_size out of range");
    if (c->max_pages_per_row <= 0) return fail(KVC_ERR_INVALID_ARGUMENT, "max_pages_per_row must be positive");
    const int64_t max_slots = (int64_t)c->max_pages_per_row * c->page_size;
    if (max_slots > (1 << 24)) return fail(KVC_ERR_UNSUPPORTED, "at most 2^24 slots per row");
    if (!c->block_table || !c->row_len || !c->slot_pos)
        return fail(KVC_ERR_INVALID_ARGUMENT, "block_table, row_len and slot_pos are required");
    if (c->dtype != KVC_F32 && c->dtype != KVC_BF16) return fail(KVC_ERR_UNSUPPORTED, "dtype must be KVC_F32 or KVC_BF16");
    if (c->head_dim != 64 && c->head_dim != 128) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (need_pools) {
        if (!c->k_pool || !c->v_pool) return fail(KVC_ERR_INVALID_ARGUMENT, "k_pool and v_pool are required");
        if (((uintptr_t)c->k_pool | (uintptr_t)c->v_pool) & 15)
            return fail(KVC_ERR_INVALID_ARGUMENT, "k_pool and v_pool must be 16-byte aligned");
        if (c->num_pages <= 0 || c->num_pages > (int64_t)INT32_MAX)
            return fail(KVC_ERR_INVALID_ARGUMENT, "num_pages out of range");
    }
    v.k_pool = c->k_pool;
    v.v_pool = c->v_pool;
    v.num_pages = c->num_pages;
    v.page_size = c->page_size;
    v.head_dim = c->head_dim;
    v.dtype = c->dtype;
    v.max_pages_per_row = c->max_pages_per_row;
    v.block_table = c->block_table;
    v.row_len = c->row_len;
    v.slot_pos = c->slot_pos;
    v.slot_label = c->slot_label;
    v.num_seqs = c->num_seqs;
    v.num_layers = c->num_layers;
    v.num_kv_heads = c->num_kv_heads;
    v.rows = (int32_t)rows;
    v.max_slots = max_slots;
    return KVC_OK;
}

kvc_status view_queries(const kvc_queries *q, const kvc::CacheView &c, kvc::QueryView &v) {
    if (!q) return fail(KVC_ERR_INVALID_ARGUMENT, "queries is NULL");
    if (!q->q || !q->lse || !q->q_pos || !q->num_q) return fail(KVC_ERR_INVALID_ARGUMENT, "query arrays are required");
    if (q->max_q <= 0 || q->max_q > (1 << 20)) return fail(KVC_ERR_INVALID_ARGUMENT, "max_q out of range");
    if (q->num_q_heads <= 0 || q->num_q_heads % c.num_kv_heads != 0)
        return fail(KVC_ERR_INVALID_ARGUMENT, "num_q_heads must be a positive multiple of num_kv_heads");
    if (((uintptr_t)q->q) & 15) return fail(KVC_ERR_INVALID_ARGUMENT, "q must be 16-byte aligned");
    v.q = q->q;
    v.lse = q->lse;
    v.q_pos = q->q_pos;
    v.num_q = q->num_q;
    v.max_q = q->max_q;
    v.num_q_heads = q->num_q_heads;
    v.group = q->num_q_heads / c.num_kv_heads;
    if (v.group > 128) return fail(KVC_ERR_UNSUPPORTED, "at most 128 query heads per KV head");
    return KVC_OK;
}

kvc_status check_params(const kvc_ratchet_params *p) {
    if (!p) return fail(KVC_ERR_INVALID_ARGUMENT, "params is NULL");
    if (p->top_k <= 0 || p->top_k > 64) return fail(KVC_ERR_UNSUPPORTED, "top_k must be in [1, 64]");
    if (p->window <= 0 || p->window > 4096 || p->stride <= 0 || p->stride > p->window)
        return fail(KVC_ERR_INVALID_ARGUMENT, "need 0 < stride <= window <= 4096");
    if (p->grow_num <= 0 || p->grow_den <= 0 || p->grow_num < p->grow_den)
        return fail(KVC_ERR_INVALID_ARGUMENT, "growth must be a ratio >= 1");
    if (p->init_budget < 0 || p->cap < p->init_budget) return fail(KVC_ERR_INVALID_ARGUMENT, "need 0 <= init_budget <= cap");
    if (p->min_points < 2) return fail(KVC_ERR_INVALID_ARGUMENT, "min_points must be at least 2");
    if (p->max_steps <= 0 || p->max_steps > (1 << 20)) return fail(KVC_ERR_INVALID_ARGUMENT, "max_steps out of range");
    return KVC_OK;
}

}  // namespace

namespace kvc {
void set_last_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}
}  // namespace kvc

extern "C" {

const char *kvc_status_string(kvc_status s) {
    switch (s) {
        case KVC_OK: return "ok";
        case KVC_ERR_INVALID_ARGUMENT: return "invalid argument";
        case KVC_ERR_UNSUPPORTED: return "unsupported";
        case KVC_ERR_CUDA: return "CUDA error";
        case KVC_ERR_DEVICE_FAULT: return "device-detected fault";
        case KVC_ERR_TIMEOUT: return "timeout";
    }
    return "unknown status";
}

const char *kvc_last_error(void) { return g_err; }

int32_t kvc_version(void) { return 1; }

kvc_status kvc_query_lse(const kvc_cache *cache, const kvc_queries *queries, int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc::QueryView q;
    kvc_status s = view_cache(cache, c, true);
    if (s != KVC_OK) return s;
    if ((s = view_queries(queries, c, q)) != KVC_OK) return s;
    if (kvc::lse_tc_supported(c, q))
        return cuda_status(kvc::launch_lse_tc(c, q, d_status, (cudaStream_t)stream), "kvc_query_lse launch");
    return cuda_status(kvc::launch_lse_simt(c, q, d_status, (cudaStream_t)stream), "kvc_query_lse launch");
}

kvc_status kvc_score_from_lse(const kvc_cache *cache, const kvc_queries *queries, float *scores, uint32_t flags,
                              int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc::QueryView q;
    kvc_status s = view_cache(cache, c, true);
    if (s != KVC_OK) return s;
    if ((s = view_queries(queries, c, q)) != KVC_OK) return s;
    if (!scores) return fail(KVC_ERR_INVALID_ARGUMENT, "scores is NULL");
    if (flags & ~(KVC_SCORE_ACCUMULATE | KVC_SCORE_COMPUTE_LSE | KVC_SCORE_SIMT))
        return fail(KVC_ERR_INVALID_ARGUMENT, "unknown flags");
    cudaStream_t st = (cudaStream_t)stream;
    if (flags & KVC_SCORE_COMPUTE_LSE) {
        const bool tc = kvc::lse_tc_supported(c, q) && !(flags & KVC_SCORE_SIMT);
        if ((s = cuda_status(tc ? kvc::launch_lse_tc(c, q, d_status, st) : kvc::launch_lse_simt(c, q, d_status, st),
                             "lse launch")) != KVC_OK)
            return s;
    }
    const bool acc = (flags & KVC_SCORE_ACCUMULATE) != 0;
    if (c.dtype == KVC_BF16 && !(flags & KVC_SCORE_SIMT)) {
        if (c.page_size != 16) return fail(KVC_ERR_UNSUPPORTED, "tensor-core scoring needs page_size 16");
        char err[256] = "";
        cudaError_t e = kvc::launch_score_tc(c, q, scores, acc, d_status, st, err, sizeof(err));
        if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "score (tensor cores): %s %s", cudaGetErrorString(e), err);
        return KVC_OK;
    }
    return cuda_status(kvc::launch_score_simt(c, q, scores, acc, d_status, st), "score (CUDA cores) launch");
}

kvc_status kvc_lrfu_update(const kvc_cache *cache, const float *scores, float *crf, float lambda, float hit_mass,
                           int32_t dt_rounds, uint32_t flags, int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, false);
    if (s != KVC_OK) return s;
    if (!scores || !crf) return fail(KVC_ERR_INVALID_ARGUMENT, "scores and crf are required");
    if (!(lambda >= 0.f) || !std::isfinite(lambda)) return fail(KVC_ERR_INVALID_ARGUMENT, "lambda must be >= 0");
    if (!(hit_mass > 0.f) || !std::isfinite(hit_mass)) return fail(KVC_ERR_INVALID_ARGUMENT, "hit_mass must be > 0");
    if (dt_rounds < 0) return fail(KVC_ERR_INVALID_ARGUMENT, "dt_rounds must be >= 0");
    if (flags & ~KVC_HIT_BINARY) return fail(KVC_ERR_INVALID_ARGUMENT, "unknown flags");
    const float decay = (float)std::exp2(-(double)lambda * (double)dt_rounds);
    return cuda_status(kvc::launch_lrfu(c, scores, crf, decay, hit_mass, (flags & KVC_HIT_BINARY) != 0, d_status,
                                        (cudaStream_t)stream),
                       "kvc_lrfu_update launch");
}

kvc_status kvc_select_budget(const kvc_cache *cache, const float *crf, const int32_t *budget,
                             uint32_t protect_label_mask, uint8_t *keep, int32_t *kept, int32_t *d_status,
                             kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, false);
    if (s != KVC_OK) return s;
    if (!crf || !budget || !keep || !kept) return fail(KVC_ERR_INVALID_ARGUMENT, "crf, budget, keep and kept are required");
    return cuda_status(kvc::launch_select(c, crf, budget, protect_label_mask, keep, kept, d_status, (cudaStream_t)stream),
                       "kvc_select_budget launch");
}

kvc_status kvc_lrfu_select(const kvc_cache *cache, const float *scores, float *crf, float lambda, float hit_mass,
                           int32_t dt_rounds, uint32_t flags, const int32_t *budget, uint32_t protect_label_mask,
                           uint8_t *keep, int32_t *kept, int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, false);
    if (s != KVC_OK) return s;
    if (!scores || !crf) return fail(KVC_ERR_INVALID_ARGUMENT, "scores and crf are required");
    if (!budget || !keep || !kept) return fail(KVC_ERR_INVALID_ARGUMENT, "budget, keep and kept are required");
    if (!(lambda >= 0.f) || !std::isfinite(lambda)) return fail(KVC_ERR_INVALID_ARGUMENT, "lambda must be >= 0");
    if (!(hit_mass > 0.f) || !std::isfinite(hit_mass)) return fail(KVC_ERR_INVALID_ARGUMENT, "hit_mass must be > 0");
    if (dt_rounds < 0) return fail(KVC_ERR_INVALID_ARGUMENT, "dt_rounds must be >= 0");
    if (flags & ~KVC_HIT_BINARY) return fail(KVC_ERR_INVALID_ARGUMENT, "unknown flags");
    const float decay = (float)std::exp2(-(double)lambda * (double)dt_rounds);
    return cuda_status(kvc::launch_lrfu_select(c, scores, crf, decay, hit_mass, (flags & KVC_HIT_BINARY) != 0, budget,
                                               protect_label_mask, keep, kept, d_status, (cudaStream_t)stream),
                       "kvc_lrfu_select launch");
}

kvc_status kvc_plan_slots(const kvc_cache *cache, const uint8_t *keep, const int32_t *kept, int32_t *move_src,
                          int32_t *move_dst, int32_t *num_moves, int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, false);
    if (s != KVC_OK) return s;
    if (!keep || !kept || !move_src || !move_dst || !num_moves)
        return fail(KVC_ERR_INVALID_ARGUMENT, "keep, kept, move_src, move_dst and num_moves are required");
    return cuda_status(kvc::launch_plan(c, keep, kept, move_src, move_dst, num_moves, d_status, (cudaStream_t)stream),
                       "kvc_plan_slots launch");
}

kvc_status kvc_select_plan(const kvc_cache *cache, const float *crf, const int32_t *budget,
                           uint32_t protect_label_mask, uint8_t *keep, int32_t *kept, int32_t *move_src,
                           int32_t *move_dst, int32_t *num_moves, int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, false);
    if (s != KVC_OK) return s;
    if (!crf || !budget || !keep || !kept) return fail(KVC_ERR_INVALID_ARGUMENT, "crf, budget, keep and kept are required");
    if (!move_src || !move_dst || !num_moves)
        return fail(KVC_ERR_INVALID_ARGUMENT, "move_src, move_dst and num_moves are required");
    return cuda_status(kvc::launch_select_plan(c, crf, budget, protect_label_mask, keep, kept, move_src, move_dst,
                                               num_moves, d_status, (cudaStream_t)stream),
                       "kvc_select_plan launch");
}

size_t kvc_compact_workspace_bytes(int32_t rows) {
    return rows < 0 ? 0 : ((size_t)rows + 1) * sizeof(int64_t);
}

kvc_status kvc_compact_pages(const kvc_cache *cache, const int32_t *move_src, const int32_t *move_dst,
                             const int32_t *num_moves, const int32_t *new_len, float *crf, int32_t *freed,
                             int64_t freed_capacity, int64_t *num_freed, void *workspace, size_t workspace_bytes,
                             int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, true);
    if (s != KVC_OK) return s;
    if (!move_src || !move_dst || !num_moves || !new_len || !num_freed)
        return fail(KVC_ERR_INVALID_ARGUMENT, "move_src, move_dst, num_moves, new_len and num_freed are required");
    if (freed_capacity < 0 || (freed_capacity > 0 && !freed))
        return fail(KVC_ERR_INVALID_ARGUMENT, "freed is NULL or freed_capacity < 0");
    if (!workspace || workspace_bytes < kvc_compact_workspace_bytes(c.rows) || ((uintptr_t)workspace & 7))
        return fail(KVC_ERR_INVALID_ARGUMENT, "workspace must be 8-byte aligned and at least %zu bytes",
                    kvc_compact_workspace_bytes(c.rows));
    const int esize = c.dtype == KVC_BF16 ? 2 : 4;
    if ((c.head_dim * esize) % 16) return fail(KVC_ERR_UNSUPPORTED, "head_dim * element size must be a multiple of 16");
    return cuda_status(kvc::launch_compact(c, move_src, move_dst, num_moves, new_len, crf, freed, freed_capacity,
                                           num_freed, static_cast<int64_t *>(workspace), d_status,
                                           (cudaStream_t)stream),
                       "kvc_compact_pages launch");
}

size_t kvc_append_workspace_bytes(int32_t rows) {
    return rows < 0 ? 0 : (2 * (size_t)rows + 2) * sizeof(int64_t);
}

kvc_status kvc_append_tokens(const kvc_cache *cache, const void *k_new, const void *v_new, const int32_t *new_pos,
                             int32_t count, uint8_t label, float *crf, int32_t *free_pages, int64_t *free_count,
                             void *workspace, size_t workspace_bytes, int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, true);
    if (s != KVC_OK) return s;
    if (count < 0) return fail(KVC_ERR_INVALID_ARGUMENT, "count must be >= 0");
    if (count == 0) return KVC_OK;
    if (!k_new || !v_new || !new_pos || !free_pages || !free_count)
        return fail(KVC_ERR_INVALID_ARGUMENT, "k_new, v_new, new_pos, free_pages and free_count are required");
    const int esize = c.dtype == KVC_BF16 ? 2 : 4;
    if ((c.head_dim * esize) % 16) return fail(KVC_ERR_UNSUPPORTED, "head_dim * element size must be a multiple of 16");
    if (((uintptr_t)k_new | (uintptr_t)v_new) & 15) return fail(KVC_ERR_INVALID_ARGUMENT, "k_new and v_new must be 16-byte aligned");
    if (!workspace || workspace_bytes < kvc_append_workspace_bytes(c.rows) || ((uintptr_t)workspace & 7))
        return fail(KVC_ERR_INVALID_ARGUMENT, "workspace must be 8-byte aligned and at least %zu bytes",
                    kvc_append_workspace_bytes(c.rows));
    return cuda_status(kvc::launch_append(c, k_new, v_new, new_pos, count, label, crf, free_pages, free_count,
                                          static_cast<int64_t *>(workspace), d_status, (cudaStream_t)stream),
                       "kvc_append_tokens launch");
}

size_t kvc_ratchet_state_bytes(int32_t num_seqs, const kvc_ratchet_params *params) {
    if (num_seqs <= 0 || check_params(params) != KVC_OK) return 0;
    return kvc::ratchet_state_bytes(num_seqs, *params);
}

kvc_status kvc_beacon_update(const void *q, const int32_t *num_q, int32_t num_seqs, int32_t num_layers,
                             int32_t num_q_heads, int32_t head_dim, int32_t max_q, kvc_dtype dtype, float *beacons,
                             int32_t *counts, int32_t num_beacons, void *beacon_q, int32_t out_max_q,
                             int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    if (!q || !num_q || !beacons || !counts) return fail(KVC_ERR_INVALID_ARGUMENT, "q, num_q, beacons and counts are required");
    if (dtype != KVC_BF16 && dtype != KVC_F32) return fail(KVC_ERR_UNSUPPORTED, "dtype must be bf16 or f32");
    if (num_seqs <= 0 || num_layers <= 0 || num_q_heads <= 0)
        return fail(KVC_ERR_INVALID_ARGUMENT, "num_seqs, num_layers and num_q_heads must be positive");
    if ((int64_t)num_seqs * num_layers * num_q_heads > INT32_MAX) return fail(KVC_ERR_UNSUPPORTED, "too many groups");
    if (head_dim <= 0 || head_dim > 256) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be in [1, 256]");
    if (num_beacons <= 0 || num_beacons > 64) return fail(KVC_ERR_UNSUPPORTED, "num_beacons must be in [1, 64]");
    if (max_q <= 0 || max_q > 65536) return fail(KVC_ERR_UNSUPPORTED, "max_q must be in [1, 65536]");
    if (beacon_q && out_max_q < num_beacons) return fail(KVC_ERR_INVALID_ARGUMENT, "out_max_q is below num_beacons");
    return cuda_status(kvc::launch_beacon(q, num_q, num_seqs, num_layers, num_q_heads, head_dim, max_q,
                                          dtype == KVC_BF16, beacons, counts, num_beacons, beacon_q, out_max_q,
                                          d_status, (cudaStream_t)stream),
                       "kvc_beacon_update launch");
}

kvc_status kvc_decode_attention(const kvc_cache *cache, const void *q, const int32_t *q_pos, int32_t num_q_heads,
                                float *out, float *lse, float *scores, uint32_t flags, int32_t *d_status,
                                kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, true);
    if (s != KVC_OK) return s;
    if (!q || !q_pos || !out || !lse) return fail(KVC_ERR_INVALID_ARGUMENT, "q, q_pos, out and lse are required");
    if (num_q_heads <= 0 || num_q_heads % c.num_kv_heads != 0)
        return fail(KVC_ERR_INVALID_ARGUMENT, "num_q_heads must be a positive multiple of num_kv_heads");
    if (flags & ~KVC_SCORE_ACCUMULATE) return fail(KVC_ERR_INVALID_ARGUMENT, "unknown flags");
    const int group = num_q_heads / c.num_kv_heads;
    if (group > 8) return fail(KVC_ERR_UNSUPPORTED, "at most 8 query heads per KV head");
    const int cluster = kvc::decode_cluster(c, group);
    if (cluster == 0)
        return fail(KVC_ERR_UNSUPPORTED, "a row of %lld slots with %d query heads per KV head exceeds the logits buffer",
                    (long long)c.max_slots, group);
    return cuda_status(kvc::launch_decode(c, q, q_pos, num_q_heads, out, lse, scores,
                                          (flags & KVC_SCORE_ACCUMULATE) != 0, d_status, (cudaStream_t)stream,
                                          cluster),
                       "kvc_decode_attention launch");
}

kvc_status kvc_step_scores(const kvc_cache *cache, const float *scores, const int32_t *step_start,
                           const int32_t *num_steps, int32_t max_steps, float beta, float *out, int32_t *d_status,
                           kvc_stream_t stream) {
    g_err[0] = 0;
    kvc::CacheView c;
    kvc_status s = view_cache(cache, c, false);
    if (s != KVC_OK) return s;
    if (!scores || !step_start || !num_steps || !out)
        return fail(KVC_ERR_INVALID_ARGUMENT, "scores, step_start, num_steps and out are required");
    if (max_steps < 1 || max_steps > 4096) return fail(KVC_ERR_UNSUPPORTED, "max_steps must be in [1, 4096]");
    if (!(beta >= 0.f && beta <= 1.f)) return fail(KVC_ERR_INVALID_ARGUMENT, "beta must be in [0, 1]");
    return cuda_status(kvc::launch_step_scores(c, scores, step_start, num_steps, max_steps, beta, out, d_status,
                                               (cudaStream_t)stream),
                       "kvc_step_scores launch");
}

kvc_status kvc_ratchet_init(void *state, int32_t *budget, int32_t num_seqs, const kvc_ratchet_params *params,
                            kvc_stream_t stream) {
    g_err[0] = 0;
    kvc_status s = check_params(params);
    if (s != KVC_OK) return s;
    if (!state || num_seqs <= 0 || num_seqs > 65535) return fail(KVC_ERR_INVALID_ARGUMENT, "state is NULL or num_seqs out of range");
    if ((uintptr_t)state & 15) return fail(KVC_ERR_INVALID_ARGUMENT, "state must be 16-byte aligned");
    return cuda_status(kvc::launch_ratchet_init(state, budget, num_seqs, *params, (cudaStream_t)stream),
                       "kvc_ratchet_init launch");
}

kvc_status kvc_confidence_ratchet(const float *logits, int32_t num_seqs, int32_t steps, int32_t vocab, void *state,
                                  int32_t *budget, float *confidence_out, const kvc_ratchet_params *params,
                                  int32_t *d_status, kvc_stream_t stream) {
    g_err[0] = 0;
    kvc_status s = check_params(params);
    if (s != KVC_OK) return s;
    if (!state || !budget || (steps > 0 && !logits)) return fail(KVC_ERR_INVALID_ARGUMENT, "logits, state and budget are required");
    if ((uintptr_t)state & 15) return fail(KVC_ERR_INVALID_ARGUMENT, "state must be 16-byte aligned");
    if (num_seqs <= 0 || num_seqs > 65535) return fail(KVC_ERR_INVALID_ARGUMENT, "num_seqs out of range");
    if (steps < 0 || steps > params->max_steps || steps > 65535)
        return fail(KVC_ERR_INVALID_ARGUMENT, "steps must be in [0, params->max_steps]");
    if (vocab <= 0 || vocab > (1 << 24)) return fail(KVC_ERR_UNSUPPORTED, "vocab must be in [1, 2^24]");
    return cuda_status(kvc::launch_ratchet(logits, num_seqs, steps, vocab, state, budget, confidence_out, *params,
                                           d_status, (cudaStream_t)stream),
                       "kvc_confidence_ratchet launch");
}

}  // extern "C"
