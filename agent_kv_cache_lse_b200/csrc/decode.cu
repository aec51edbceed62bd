// One decode step of paged attention with the eviction scores folded in.
//
// "ActKV Dissected", Component 3: the softmax log-sum-exp is a byproduct of paged
// attention, so the current query's attention probabilities are its logits minus the LSE,
// with no gather of the attention matrix and no recompute.  Here the decode kernel does it
// itself.  For each row (sequence, layer, KV head), the G query heads of its group and the
// row's keys at or before the query's position:
//   l[g, i] = q_g . k_i / sqrt(D),  lse[g] = log sum_i exp(l[g, i]),
//   out[g] = sum_i exp(l[g, i] - lse[g]) v_i,  scores[i] (+)= sum_g exp(l[g, i] - lse[g]).
//
// One cluster of C CTAs per row; each CTA owns a contiguous slice of the row's slots:
//   A. logits of the slice into shared memory and per-head slice maxima.  A warp takes
//      KW = 32 / (D/8) keys per step, a lane 8 elements of D (one 16-byte load), and U steps
//      are loaded before any is used, so that enough bytes are in flight to cover HBM latency;
//   B. the cluster maximum M_g through distributed shared memory; p = exp(l - M_g) in place
//      of the logits, per-head slice sums;
//   C. the slice's partial output sum_i p[g, i] v_i with the same key mapping, reduced over a
//      warp's key lanes by shuffles, then over the warps in order;
//   D. every CTA sums the cluster's per-head sums S_g in rank order; the leader adds the
//      partial outputs in rank order and writes out = O / S and lse = M + log S; each CTA adds
//      sum_g p[g, i] / S_g to its slice's scores.
// Every sum runs in a fixed order, so results repeat bit for bit from run to run.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 8;
constexpr int kMaxCluster = 8;
constexpr int kMaxD = 128;
constexpr int kUnroll = 4;
constexpr size_t kSmemBudget = 200 * 1024;
constexpr size_t kTwoPerSm = 100 * 1024;  // dynamic bytes under which two CTAs share an SM

struct DecodeArgs {
    CacheView c;
    const void *q;        // [S][L][Hq][D], cache dtype
    const int32_t *q_pos; // [S]
    int32_t num_q_heads, group;
    float *out;           // [S][L][Hq][D]
    float *lse;           // [S][L][Hq]
    float *scores;        // [rows][max_slots] or null
    int32_t accumulate;
    int32_t slice_cap;    // slots per CTA the logits buffer holds
    float scale;          // 1 / sqrt(D)
    int32_t *status;
};

struct DecodeShared {
    float pmax[kMaxGroup];          // published per-head slice maxima
    float psum[kMaxGroup];          // published per-head slice sums
    float pout[kMaxGroup * kMaxD];  // published partial outputs [g][d]
    float red[kWarps][kMaxGroup];
    float M[kMaxGroup], S[kMaxGroup];
    int32_t bad;
};

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(h[t]);
        x[2 * t] = f.x;
        x[2 * t + 1] = f.y;
    }
}

__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <typename T, int D, int GM>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(DecodeArgs a) {
    constexpr int LK = D / 8;        // lanes per key
    constexpr int KW = 32 / LK;      // keys per warp step
    constexpr int STEP = KW * kUnroll;
    extern __shared__ __align__(16) float smem_f[];
    __shared__ DecodeShared sh;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank(), C = (int)cl.num_blocks();
    const int row = blockIdx.x / C;
    const CacheView &c = a.c;
    const int G = a.group, Hkv = c.num_kv_heads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kslot = lane / LK, sub = lane % LK;
    const int seq = row / (c.num_layers * Hkv), layer = (row / Hkv) % c.num_layers, kvh = row % Hkv;
    float *qs = smem_f;                                   // [GM][D]
    float *lg = qs + GM * D;                              // [GM][slice_cap]: logits, then probabilities
    float *part = lg + (size_t)GM * a.slice_cap;          // [kWarps][G][D] partial outputs

    int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (rank == 0 && tid == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        n = 0;  // the row still takes part in the cluster steps, with no keys
    }
    const int per = (n + C - 1) / C;
    const int lo = min(n, rank * per), hi = min(n, lo + per), cnt = hi - lo;
    const int qpos = a.q_pos[seq];
    const int64_t hbase = (int64_t)(seq * c.num_layers + layer) * a.num_q_heads + kvh * G;  // the group's first head
    for (int i = tid; i < GM * D; i += kThreads)
        qs[i] = i < G * D ? static_cast<float>(static_cast<const T *>(a.q)[hbase * D + i]) : 0.f;
    if (tid == 0) sh.bad = 0;
    __syncthreads();

    const T *kp = static_cast<const T *>(c.k_pool);
    const T *vp = static_cast<const T *>(c.v_pool);
    const int32_t *bt = c.block_table + (int64_t)row * c.max_pages_per_row;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots + lo;
    // element offset of this lane's 8 values of local slot il in a pool; -1 when the slot is past
    // the slice, hidden by the causal mask or on an unreadable page
    auto key_off = [&](int il, bool flag) -> int64_t {
        if (il >= cnt || pos[il] > qpos) return -1;
        const int i = lo + il;
        const int page = bt[i / c.page_size];
        if (page < 0 || page >= c.num_pages) {
            if (flag) sh.bad = 1;
            return -1;
        }
        return ((int64_t)page * c.page_size + i % c.page_size) * D + sub * 8;
    };

    // A. logits and per-head slice maxima
    float qr[GM][8];
#pragma unroll
    for (int g = 0; g < GM; ++g)
#pragma unroll
        for (int t = 0; t < 8; ++t) qr[g][t] = qs[g * D + sub * 8 + t];
    float hmax[GM];
#pragma unroll
    for (int g = 0; g < GM; ++g) hmax[g] = -INFINITY;
    for (int i0 = warp * STEP; i0 < cnt; i0 += kWarps * STEP) {
        int64_t off[kUnroll];
        float x[kUnroll][8];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) off[u] = key_off(i0 + u * KW + kslot, true);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (off[u] >= 0) load8(kp + off[u], x[u]);
            else {
#pragma unroll
                for (int t = 0; t < 8; ++t) x[u][t] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int il = i0 + u * KW + kslot;
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                float acc = qr[g][0] * x[u][0];
#pragma unroll
                for (int t = 1; t < 8; ++t) acc = fmaf(qr[g][t], x[u][t], acc);
#pragma unroll
                for (int o = LK / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                const float l = off[u] >= 0 ? acc * a.scale : -INFINITY;
                if (il < cnt && sub == 0) lg[(size_t)g * a.slice_cap + il] = l;
                hmax[g] = fmaxf(hmax[g], l);
            }
        }
    }
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        const float m = warp_max(hmax[g]);
        if (lane == 0) sh.red[warp][g] = m;
    }
    __syncthreads();
    if (tid < GM) {
        float m = -INFINITY;
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sh.red[w][tid]);
        sh.pmax[tid] = m;
    }
    cl.sync();

    // B. cluster maxima, probabilities against them, per-head slice sums
    if (tid < GM) {
        float m = -INFINITY;
        for (int r = 0; r < C; ++r) m = fmaxf(m, cl.map_shared_rank(&sh, r)->pmax[tid]);
        sh.M[tid] = m;
    }
    __syncthreads();
    float hs[GM];
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        hs[g] = 0.f;
        const float m = sh.M[g];
        float *e = lg + (size_t)g * a.slice_cap;
        for (int i = tid; i < cnt; i += kThreads) {
            const float p = m == -INFINITY ? 0.f : expf(e[i] - m);
            e[i] = p;
            hs[g] += p;
        }
    }
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        const float s = warp_sum(hs[g]);
        if (lane == 0) sh.red[warp][g] = s;
    }
    __syncthreads();
    if (tid < GM) {
        float s = 0.f;
        for (int w = 0; w < kWarps; ++w) s += sh.red[w][tid];
        sh.psum[tid] = s;
    }

    // C. the slice's partial output
    float o8[GM][8];
#pragma unroll
    for (int g = 0; g < GM; ++g)
#pragma unroll
        for (int t = 0; t < 8; ++t) o8[g][t] = 0.f;
    for (int i0 = warp * STEP; i0 < cnt; i0 += kWarps * STEP) {
        int64_t off[kUnroll];
        float x[kUnroll][8];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) off[u] = key_off(i0 + u * KW + kslot, false);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (off[u] >= 0) load8(vp + off[u], x[u]);
            else {
#pragma unroll
                for (int t = 0; t < 8; ++t) x[u][t] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int il = min(i0 + u * KW + kslot, cnt - 1);  // past the slice: x is zero
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                const float p = lg[(size_t)g * a.slice_cap + il];
#pragma unroll
                for (int t = 0; t < 8; ++t) o8[g][t] = fmaf(p, x[u][t], o8[g][t]);
            }
        }
    }
#pragma unroll
    for (int g = 0; g < GM; ++g)
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int o = LK; o < 32; o <<= 1) o8[g][t] += __shfl_xor_sync(0xffffffffu, o8[g][t], o);
    if (kslot == 0) {
        float *mine = part + (size_t)warp * G * D + sub * 8;
#pragma unroll
        for (int g = 0; g < GM; ++g)
            if (g < G)
#pragma unroll
                for (int t = 0; t < 8; ++t) mine[g * D + t] = o8[g][t];
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kThreads) {
        float s = 0.f;
        for (int w = 0; w < kWarps; ++w) s += part[(size_t)w * G * D + e];
        sh.pout[e] = s;
    }
    cl.sync();

    // D. combine
    if (tid < GM) {
        float s = 0.f;
        for (int r = 0; r < C; ++r) s += cl.map_shared_rank(&sh, r)->psum[tid];
        sh.S[tid] = s;
    }
    __syncthreads();
    if (rank == 0) {
        for (int e = tid; e < G * D; e += kThreads) {
            float o = 0.f;
            for (int r = 0; r < C; ++r) o += cl.map_shared_rank(&sh, r)->pout[e];
            const float s = sh.S[e / D];
            a.out[hbase * D + e] = s > 0.f ? o / s : 0.f;
        }
        if (tid < G) a.lse[hbase + tid] = sh.S[tid] > 0.f ? sh.M[tid] + logf(sh.S[tid]) : -INFINITY;
        if (tid == 0) {
            bool bad = false;
            for (int r = 0; r < C; ++r) bad |= cl.map_shared_rank(&sh, r)->bad != 0;
            if (bad) report(a.status, KVC_DEV_BAD_PAGE, row);
        }
    }
    if (a.scores) {
        float inv[GM];
#pragma unroll
        for (int g = 0; g < GM; ++g) inv[g] = (g < G && sh.S[g] > 0.f) ? 1.f / sh.S[g] : 0.f;
        float *sc = a.scores + (int64_t)row * c.max_slots + lo;
        for (int i = tid; i < cnt; i += kThreads) {
            float v = 0.f;
#pragma unroll
            for (int g = 0; g < GM; ++g) v = fmaf(lg[(size_t)g * a.slice_cap + i], inv[g], v);
            sc[i] = a.accumulate ? sc[i] + v : v;
        }
    }
    cl.sync();  // peers may still be reading this CTA's shared memory
}

int group_bound(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

size_t smem_bytes(const CacheView &c, int G, int C) {
    const int GM = group_bound(G);
    return (size_t)GM * c.head_dim * 4 + (size_t)kWarps * G * c.head_dim * 4 +
           (size_t)GM * ((c.max_slots + C - 1) / C) * 4;
}

template <typename T, int D, int GM>
cudaError_t launch_t(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, int C) {
    const int G = num_q_heads / c.num_kv_heads;
    const size_t smem = smem_bytes(c, G, C);
    const int cap = (int)((c.max_slots + C - 1) / C);
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D, GM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    DecodeArgs a{c, q, q_pos, num_q_heads, G, out, lse, scores, accumulate ? 1 : 0, cap,
                 (float)(1.0 / std::sqrt((double)D)), status};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c.rows * C));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<T, D, GM>, a);
}

template <typename T, int D>
cudaError_t launch_g(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, int C) {
    switch (group_bound(num_q_heads / c.num_kv_heads)) {
        case 1: return launch_t<T, D, 1>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C);
        case 2: return launch_t<T, D, 2>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C);
        case 4: return launch_t<T, D, 4>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C);
        default: return launch_t<T, D, 8>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C);
    }
}

}  // namespace

int decode_cluster(const CacheView &c, int32_t group) {
    if (group < 1 || group > kMaxGroup) return 0;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // the smallest cluster whose CTAs fit two to an SM and whose grid holds two CTAs per SM;
    // else, for long rows, the smallest whose CTAs fit at all
    int C = 1;
    while (C < kMaxCluster && (smem_bytes(c, group, C) > kTwoPerSm || (int64_t)c.rows * C < 2 * (int64_t)sms)) C <<= 1;
    return smem_bytes(c, group, C) <= kSmemBudget ? C : 0;
}

cudaError_t launch_decode(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                          float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, int C) {
    const bool bf16 = c.dtype == KVC_BF16;
    if (c.head_dim == 64)
        return bf16 ? launch_g<__nv_bfloat16, 64>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C)
                    : launch_g<float, 64>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C);
    return bf16 ? launch_g<__nv_bfloat16, 128>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C)
                : launch_g<float, 128>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, C);
}

}  // namespace kvc
