// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kvc.h"

namespace kvc {

// Host-side lookups done once per device instead of on every call.
constexpr int kMaxDevices = 64;

// SM count of the current device.
inline int device_sms() {
    static int cache[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    int &v = cache[dev & (kMaxDevices - 1)];
    if (v == 0) {
        int sms = 148;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) v = sms;
        else return sms;
    }
    return v;
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the current device; `done` (one array per
// kernel, kMaxDevices entries, zero-initialised) remembers what each device was given, so the attribute is set
// only when a call needs more than before.
inline cudaError_t dyn_smem_at_least(const void *kernel, size_t bytes, int *done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int &have = done[dev & (kMaxDevices - 1)];
    if ((size_t)have >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) have = (int)bytes;
    return e;
}

// Geometry and pointers resolved once on the host for a call.
struct CacheView {
    const void *k_pool;
    const void *v_pool;
    int64_t num_pages;
    int32_t page_size, head_dim, dtype, max_pages_per_row;
    int32_t *block_table;
    int32_t *row_len;
    int32_t *slot_pos;
    uint8_t *slot_label;
    int32_t num_seqs, num_layers, num_kv_heads;
    int32_t rows;
    int64_t max_slots;
};

struct QueryView {
    const void *q;
    float *lse;
    const int32_t *q_pos;
    const int32_t *num_q;
    int32_t max_q, num_q_heads, group;
};

// Each launcher enqueues its kernels on `stream` and returns cudaGetLastError().
cudaError_t launch_score_simt(const CacheView &c, const QueryView &q, float *scores, bool accumulate,
                              int32_t *status, cudaStream_t stream);
cudaError_t launch_lse_simt(const CacheView &c, const QueryView &q, int32_t *status, cudaStream_t stream);
cudaError_t launch_score_tc(const CacheView &c, const QueryView &q, float *scores, bool accumulate,
                            int32_t *status, cudaStream_t stream, char *err, size_t errlen);
// Tensor-core LSE pass (bf16, head_dim 64 or 128, group size <= 128).
bool lse_tc_supported(const CacheView &c, const QueryView &q);
cudaError_t launch_lse_tc(const CacheView &c, const QueryView &q, int32_t *status, cudaStream_t stream);
cudaError_t launch_lrfu(const CacheView &c, const float *scores, float *crf, float decay, float hit_mass,
                        bool binary, int32_t *status, cudaStream_t stream);
cudaError_t launch_select(const CacheView &c, const float *crf, const int32_t *budget, uint32_t protect,
                          uint8_t *keep, int32_t *kept, int32_t *status, cudaStream_t stream);
cudaError_t launch_lrfu_select(const CacheView &c, const float *scores, float *crf, float decay, float hit_mass,
                               bool binary, const int32_t *budget, uint32_t protect, uint8_t *keep, int32_t *kept,
                               int32_t *status, cudaStream_t stream);
cudaError_t launch_plan(const CacheView &c, const uint8_t *keep, const int32_t *kept, int32_t *move_src,
                        int32_t *move_dst, int32_t *num_moves, int32_t *status, cudaStream_t stream);
cudaError_t launch_select_plan(const CacheView &c, const float *crf, const int32_t *budget, uint32_t protect,
                               uint8_t *keep, int32_t *kept, int32_t *move_src, int32_t *move_dst,
                               int32_t *num_moves, int32_t *status, cudaStream_t stream);
cudaError_t launch_compact(const CacheView &c, const int32_t *move_src, const int32_t *move_dst,
                           const int32_t *num_moves, const int32_t *new_len, float *crf, int32_t *freed,
                           int64_t freed_capacity, int64_t *num_freed, int64_t *row_offsets,
                           int32_t *status, cudaStream_t stream);
cudaError_t launch_append(const CacheView &c, const void *k_new, const void *v_new, const int32_t *new_pos,
                          int32_t count, uint8_t label, float *crf, int32_t *free_pages, int64_t *free_count,
                          int64_t *ws, int32_t *status, cudaStream_t stream);
cudaError_t launch_beacon(const void *q, const int32_t *num_q, int32_t num_seqs, int32_t num_layers,
                          int32_t num_q_heads, int32_t head_dim, int32_t max_q, bool bf16, float *beacons,
                          int32_t *counts, int32_t num_beacons, void *beacon_q, int32_t out_max_q, int32_t *status,
                          cudaStream_t stream);
// Cluster size the decode kernel uses for this cache and group size; 0 when a row's logits
// do not fit the shared memory of a cluster of 8 CTAs.
int decode_cluster(const CacheView &c, int32_t group);
cudaError_t launch_decode(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                          float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream,
                          int cluster);
cudaError_t launch_step_scores(const CacheView &c, const float *scores, const int32_t *step_start,
                               const int32_t *num_steps, int32_t max_steps, float beta, float *out, int32_t *status,
                               cudaStream_t stream);
cudaError_t launch_ratchet_init(void *state, int32_t *budget, int32_t num_seqs, const kvc_ratchet_params &p,
                                cudaStream_t stream);
cudaError_t launch_ratchet(const float *logits, int32_t num_seqs, int32_t steps, int32_t vocab, void *state,
                           int32_t *budget, float *conf_out, const kvc_ratchet_params &p, int32_t *status,
                           cudaStream_t stream);

size_t ratchet_state_bytes(int32_t num_seqs, const kvc_ratchet_params &p);

// Sets the thread-local message returned by kvc_last_error().
void set_last_error(const char *fmt, ...);

}  // namespace kvc
