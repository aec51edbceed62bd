// CUDA-core scoring and LSE kernels.
//
// Scoring recovers each query column's attention probabilities from the LSE the
// attention produced, p = exp(q.k / sqrt(D) - lse), and tallies them per cached
// entry over the query set and the GQA group ("ActKV Dissected", Component 3 and
// Component 1).  This path computes in fp32 on CUDA cores: it serves fp32 caches
// (where a TF32 tensor-core product would cost ~1e-3 of logit accuracy) and, on
// request, bf16 caches as a cross-check of the tensor-core path.
//
// The LSE kernel stands in for the softmax denominator a paged-attention kernel
// emits; beacon queries ("BeaconKV", Key ideas) have no such byproduct.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kTileKeys = 128;   // keys per CTA in the score kernel (one per thread)
constexpr int kColChunk = 16;    // query columns staged in shared memory at a time

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

struct ScoreSimtArgs {
    CacheView c;
    QueryView q;
    float *scores;
    int32_t *status;
    int accumulate;
    float scale;  // 1/sqrt(D)
};

// Resolve the physical page of logical slot i of a row; -1 and report when invalid.
__device__ __forceinline__ int64_t slot_page(const CacheView &c, int row, int i, int32_t *status) {
    const int32_t p = c.block_table[(int64_t)row * c.max_pages_per_row + i / c.page_size];
    if (p < 0 || p >= c.num_pages) {
        report(status, KVC_DEV_BAD_PAGE, row);
        return -1;
    }
    return p;
}

template <typename T, int D>
__global__ void __launch_bounds__(kTileKeys) score_simt_kernel(ScoreSimtArgs a) {
    const int row = blockIdx.y;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (blockIdx.x == 0 && threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const int tile0 = blockIdx.x * kTileKeys;
    if (tile0 >= n) return;
    const int per_seq = c.num_layers * c.num_kv_heads;
    const int seq = row / per_seq, layer = (row / c.num_kv_heads) % c.num_layers, kvh = row % c.num_kv_heads;
    const int G = a.q.group, Hq = a.q.num_q_heads;
    const int nq = min(a.q.num_q[seq], a.q.max_q);
    const int ncols = nq * G;

    const int i = tile0 + threadIdx.x;
    bool valid = i < n;
    float k[D];
    int32_t kpos = 0;
    if (valid) {
        const int64_t page = slot_page(c, row, i, a.status);
        valid = page >= 0;
        if (valid) {
            const T *kp = static_cast<const T *>(c.k_pool) + (page * c.page_size + i % c.page_size) * D;
#pragma unroll
            for (int d = 0; d < D; ++d) k[d] = to_f<T>(kp[d]);
            kpos = c.slot_pos[(int64_t)row * c.max_slots + i];
        }
    }

    __shared__ float qs[kColChunk][D];
    __shared__ float ls[kColChunk];
    __shared__ int32_t ps[kColChunk];
    const T *qbase = static_cast<const T *>(a.q.q) + ((int64_t)(seq * c.num_layers + layer) * a.q.max_q) * Hq * D;
    const float *lbase = a.q.lse + ((int64_t)(seq * c.num_layers + layer) * Hq) * a.q.max_q;
    float acc = 0.f;
    for (int c0 = 0; c0 < ncols; c0 += kColChunk) {
        __syncthreads();
        for (int e = threadIdx.x; e < kColChunk * D; e += blockDim.x) {
            const int cc = e / D, d = e % D, col = c0 + cc;
            float v = 0.f;
            if (col < ncols) {
                const int j = col / G, g = col % G;
                v = to_f<T>(qbase[((int64_t)j * Hq + kvh * G + g) * D + d]);
            }
            qs[cc][d] = v;
        }
        for (int cc = threadIdx.x; cc < kColChunk; cc += blockDim.x) {
            const int col = c0 + cc;
            float l = -INFINITY;
            int32_t p = -1;
            if (col < ncols) {
                const int j = col / G, g = col % G;
                l = lbase[(int64_t)(kvh * G + g) * a.q.max_q + j];
                p = a.q.q_pos[(int64_t)seq * a.q.max_q + j];
                if (!(l == -INFINITY || is_finite(l))) {
                    report(a.status, KVC_DEV_NONFINITE, row);
                    l = -INFINITY;
                }
            }
            ls[cc] = l;
            ps[cc] = p;
        }
        __syncthreads();
        if (valid) {
            const int lim = min(kColChunk, ncols - c0);
            for (int cc = 0; cc < lim; ++cc) {
                if (ps[cc] < kpos || ls[cc] == -INFINITY) continue;
                float dot = 0.f;
#pragma unroll
                for (int d = 0; d < D; ++d) dot = fmaf(k[d], qs[cc][d], dot);
                acc += expf(dot * a.scale - ls[cc]);
            }
        }
    }
    if (valid) {
        float *dst = a.scores + (int64_t)row * c.max_slots + i;
        *dst = a.accumulate ? *dst + acc : acc;
    }
}

// ---------------------------------------------------------------------------
// LSE of every query column over its row's visible keys.
// CTA = (row, chunk of kLseCols columns); threads stride over keys with an online
// (max, sum) per column, then combine across the CTA.
// ---------------------------------------------------------------------------
constexpr int kLseCols = 16;
constexpr int kLseThreads = 256;

struct LseArgs {
    CacheView c;
    QueryView q;
    int32_t *status;
    float scale;
};

template <typename T, int D>
__global__ void __launch_bounds__(kLseThreads) lse_simt_kernel(LseArgs a) {
    const int row = blockIdx.y;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    const int per_seq = c.num_layers * c.num_kv_heads;
    const int seq = row / per_seq, layer = (row / c.num_kv_heads) % c.num_layers, kvh = row % c.num_kv_heads;
    const int G = a.q.group, Hq = a.q.num_q_heads;
    const int nq = min(a.q.num_q[seq], a.q.max_q);
    const int ncols = nq * G;
    const int c0 = blockIdx.x * kLseCols;
    if (c0 >= ncols) return;
    if (n < 0 || n > c.max_slots) {
        if (blockIdx.x == 0 && threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    __shared__ float qs[kLseCols][D];
    __shared__ int32_t ps[kLseCols];
    __shared__ float red_m[kLseThreads / 32][kLseCols];
    __shared__ float red_s[kLseThreads / 32][kLseCols];
    const T *qbase = static_cast<const T *>(a.q.q) + ((int64_t)(seq * c.num_layers + layer) * a.q.max_q) * Hq * D;
    for (int e = threadIdx.x; e < kLseCols * D; e += blockDim.x) {
        const int cc = e / D, d = e % D, col = c0 + cc;
        float v = 0.f;
        if (col < ncols) {
            const int j = col / G, g = col % G;
            v = to_f<T>(qbase[((int64_t)j * Hq + kvh * G + g) * D + d]);
        }
        qs[cc][d] = v;
    }
    for (int cc = threadIdx.x; cc < kLseCols; cc += blockDim.x) {
        const int col = c0 + cc;
        ps[cc] = col < ncols ? a.q.q_pos[(int64_t)seq * a.q.max_q + col / G] : INT32_MIN;
    }
    __syncthreads();
    float m[kLseCols], s[kLseCols];
#pragma unroll
    for (int cc = 0; cc < kLseCols; ++cc) {
        m[cc] = -INFINITY;
        s[cc] = 0.f;
    }
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int32_t p = c.block_table[(int64_t)row * c.max_pages_per_row + i / c.page_size];
        if (p < 0 || p >= c.num_pages) {
            report(a.status, KVC_DEV_BAD_PAGE, row);
            continue;
        }
        const T *kp = static_cast<const T *>(c.k_pool) + ((int64_t)p * c.page_size + i % c.page_size) * D;
        float k[D];
#pragma unroll
        for (int d = 0; d < D; ++d) k[d] = to_f<T>(kp[d]);
        const int32_t kpos = c.slot_pos[(int64_t)row * c.max_slots + i];
#pragma unroll
        for (int cc = 0; cc < kLseCols; ++cc) {
            if (ps[cc] < kpos) continue;
            float dot = 0.f;
#pragma unroll
            for (int d = 0; d < D; ++d) dot = fmaf(k[d], qs[cc][d], dot);
            const float x = dot * a.scale;
            if (x > m[cc]) {
                s[cc] = s[cc] * expf(m[cc] - x) + 1.f;
                m[cc] = x;
            } else {
                s[cc] += expf(x - m[cc]);
            }
        }
    }
    // combine within warps, then across warps
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int cc = 0; cc < kLseCols; ++cc) {
        float mm = m[cc], ss = s[cc];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, mm, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, ss, o);
            const float mx = fmaxf(mm, m2);
            if (mx == -INFINITY) {
                ss = 0.f;
            } else {
                ss = ss * expf(mm - mx) + s2 * expf(m2 - mx);
            }
            mm = mx;
        }
        if (lane == 0) {
            red_m[w][cc] = mm;
            red_s[w][cc] = ss;
        }
    }
    __syncthreads();
    if (threadIdx.x < kLseCols) {
        const int cc = threadIdx.x, col = c0 + cc;
        float mx = -INFINITY;
        for (int ww = 0; ww < kLseThreads / 32; ++ww) mx = fmaxf(mx, red_m[ww][cc]);
        double tot = 0.0;
        if (mx != -INFINITY)
            for (int ww = 0; ww < kLseThreads / 32; ++ww) tot += (double)red_s[ww][cc] * exp((double)red_m[ww][cc] - mx);
        if (col < ncols) {
            const int j = col / G, g = col % G;
            float *dst = a.q.lse + ((int64_t)(seq * c.num_layers + layer) * Hq + kvh * G + g) * a.q.max_q + j;
            *dst = mx == -INFINITY ? -INFINITY : (float)((double)mx + log(tot));
        }
    }
}

template <typename T, int D>
cudaError_t launch_score_simt_t(const CacheView &c, const QueryView &q, float *scores, bool accumulate,
                                int32_t *status, cudaStream_t stream) {
    ScoreSimtArgs a{c, q, scores, status, accumulate ? 1 : 0, (float)(1.0 / sqrt((double)D))};
    dim3 grid((unsigned)((c.max_slots + kTileKeys - 1) / kTileKeys), (unsigned)c.rows);
    score_simt_kernel<T, D><<<grid, kTileKeys, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_lse_simt_t(const CacheView &c, const QueryView &q, int32_t *status, cudaStream_t stream) {
    LseArgs a{c, q, status, (float)(1.0 / sqrt((double)D))};
    dim3 grid((unsigned)((q.max_q * q.group + kLseCols - 1) / kLseCols), (unsigned)c.rows);
    lse_simt_kernel<T, D><<<grid, kLseThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_simt(const CacheView &c, const QueryView &q, float *scores, bool accumulate,
                              int32_t *status, cudaStream_t stream) {
    const bool bf = c.dtype == KVC_BF16;
    if (c.head_dim == 64)
        return bf ? launch_score_simt_t<__nv_bfloat16, 64>(c, q, scores, accumulate, status, stream)
                  : launch_score_simt_t<float, 64>(c, q, scores, accumulate, status, stream);
    return bf ? launch_score_simt_t<__nv_bfloat16, 128>(c, q, scores, accumulate, status, stream)
              : launch_score_simt_t<float, 128>(c, q, scores, accumulate, status, stream);
}

cudaError_t launch_lse_simt(const CacheView &c, const QueryView &q, int32_t *status, cudaStream_t stream) {
    const bool bf = c.dtype == KVC_BF16;
    if (c.head_dim == 64)
        return bf ? launch_lse_simt_t<__nv_bfloat16, 64>(c, q, status, stream)
                  : launch_lse_simt_t<float, 64>(c, q, status, stream);
    return bf ? launch_lse_simt_t<__nv_bfloat16, 128>(c, q, status, stream)
              : launch_lse_simt_t<float, 128>(c, q, status, stream);
}

}  // namespace kvc
