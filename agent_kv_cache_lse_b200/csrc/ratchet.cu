// Confidence monitor and one-way budget ratchet.
//
// "ActKV Dissected", Component 2 (and Summary, Lineage): the budget follows the
// model's hesitation.  Per decode step, the confidence is the average negative
// log-probability of the top-20 tokens, c_t = LSE(z_t) - mean(top-20 z_t); token
// confidences are min-pooled over sliding windows (64 wide, stride 8) into a
// trajectory-level series; a linear fit with negative slope means the budget is too
// small and grows it by 1.75x (initial 512, cap 30,000); it never shrinks.
//
// Launch A (confidence): a cluster of kCluster CTAs per (sequence, step) row of
//   logits, each CTA a slice of the vocabulary, read straight from global memory with
//   16-byte loads (no staging: the logits of a round do not fit in the shared memory of
//   the GPU, so staging would need a second wave of CTAs).  Pass 1 keeps a running
//   (max, sum of exp) per thread; the k-th largest of the warps' top-4 per-thread
//   maxima is a lower bound for the slice's k-th largest logit.  Pass 2 re-reads the
//   slice (from L2) for the values at or above that bound (a few dozen), which a warp
//   bitonic network sorts; when more than 64 qualify (many equal logits) an exact radix
//   search over the slice takes over.  The leader CTA merges the cluster's (max, sum)
//   pairs and sorted top-k lists through distributed shared memory into c_t.
// Launch B (ratchet): one warp per sequence pools the newly completed windows,
//   updates the least-squares sums, evaluates the fit once and moves the budget.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTopK = 64;

size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

struct RatchetLayout {
    size_t state_bytes;  // num_seqs * sizeof(kvc_ratchet_seq_state), 16-aligned
    int hist_len;        // window - 1 + max_steps
};

RatchetLayout layout_of(int32_t num_seqs, const kvc_ratchet_params &p) {
    RatchetLayout l;
    l.state_bytes = align16((size_t)num_seqs * sizeof(kvc_ratchet_seq_state));
    l.hist_len = p.window - 1 + p.max_steps;
    return l;
}

struct ConfArgs {
    const float *logits;
    int32_t steps, vocab, chunk;
    int32_t top_k;
    int32_t vec;        // rows and slices 16-byte aligned: 16-byte loads
    float *hist;        // [seqs][hist_len]
    int32_t hist_len, window;
    float *conf_out;    // [seqs][steps] or null
    int32_t *status;
};

// 2^x by the MUFU unit (ex2.approx, relative error ~2^-22): ample for the log-sum-exp of a step.
__device__ __forceinline__ float exp2f_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Descending sort of 64 values held two per lane (lane l holds v[0] = x[l], v[1] = x[l + 32]) with a
// bitonic network over the warp.
__device__ __forceinline__ void warp_sort64_desc(float &a, float &b) {
    const int lane = threadIdx.x & 31;
    // element index e = lane (a) and lane + 32 (b)
    for (int k = 2; k <= 64; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {
                // partners are a and b of the same lane
                const bool desc = (lane & k) == 0;  // k == 64 here: whole array descending
                const float hi = fmaxf(a, b), lo = fminf(a, b);
                a = desc ? hi : lo;
                b = desc ? lo : hi;
            } else {
                const float pa = __shfl_xor_sync(0xffffffffu, a, j);
                const float pb = __shfl_xor_sync(0xffffffffu, b, j);
                const bool lower = (lane & j) == 0;
                const bool da = (lane & k) == 0, db = ((lane + 32) & k) == 0;
                a = (lower == da) ? fmaxf(a, pa) : fminf(a, pa);
                b = (lower == db) ? fmaxf(b, pb) : fminf(b, pb);
            }
        }
    }
}

struct ConfShared {
    float cand[64];
    float topk[kMaxTopK];        // this CTA's top-k, descending (-inf pads a short slice)
    float wtop[32];              // top-4 per warp of the per-thread maxima
    float red_f[32];
    double red_d[32];
    int red_i[32];
    unsigned int hist[256];      // exact fallback: digit counts
    uint32_t fb_prefix, fb_pmask;
    int fb_above, fb_remaining;
    float cmax;
    double csum;
    int ncand;
    int nbad;
};

// Running (max m, sum s of exp(z - m)) of a thread: one exponential per value, two when the max moves.
struct RunLse {
    float m = -INFINITY, s = 0.f;
    int bad = 0;
    __device__ __forceinline__ void add(float z) {
        if (!is_finite(z)) {
            if (z != -INFINITY) bad = 1;  // -inf contributes nothing; NaN and +inf are errors
            return;
        }
        if (z > m) {
            s = s * exp2f_fast((m - z) * 1.4426950408889634f) + 1.f;
            m = z;
        } else {
            s += exp2f_fast((z - m) * 1.4426950408889634f);
        }
    }
};

__global__ void __launch_bounds__(kThreads) confidence_kernel(ConfArgs a) {
    __shared__ ConfShared sh;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int step = blockIdx.y, seq = blockIdx.z;
    const int K = a.top_k;
    const float *row = a.logits + ((int64_t)seq * a.steps + step) * a.vocab;
    const int lo = min(a.vocab, rank * a.chunk), hi = min(a.vocab, lo + a.chunk);
    const int cnt = hi - lo;
    const float *z = row + lo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) sh.ncand = 0;
    // the slice as 16-byte vectors (a.vec: the slice starts 16-byte aligned) plus a scalar tail
    const int n4 = a.vec ? cnt >> 2 : 0;
    const float4 *z4 = reinterpret_cast<const float4 *>(z);

    // pass 1: running (max, sum of exp) per thread, four vectors in flight
    RunLse r;
    for (int i = tid; i < n4; i += 4 * kThreads) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = i + u * kThreads < n4 ? z4[i + u * kThreads] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            r.add(v[u].x);
            r.add(v[u].y);
            r.add(v[u].z);
            r.add(v[u].w);
        }
    }
    for (int i = 4 * n4 + tid; i < cnt; i += kThreads) r.add(z[i]);
    const float tmax = r.m;

    // lower bound tau0 for the slice's k-th largest: the k-th largest of the warps' top-4 per-thread maxima
    // (32 distinct values of the slice)
    {
        float cur = tmax;
        bool taken = false;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float mq = taken ? -INFINITY : cur;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
            const unsigned who = __ballot_sync(0xffffffffu, !taken && cur == mq);
            if (lane == __ffs(who) - 1) taken = true;
            if (lane == 0) sh.wtop[4 * warp + q] = mq;
        }
    }
    const float cmax = block_max(tmax, sh.red_f);  // also orders the wtop writes
    const double csum = block_sum<double>(cmax == -INFINITY ? 0.0 : (double)r.s * exp((double)r.m - (double)cmax),
                                          sh.red_d);
    const int bad = block_or(r.bad, sh.red_i);
    float tau0 = -INFINITY;
    if (cnt >= K && K <= 4 * kWarps) {
        // every warp ranks the 32 values for the bound; identical in all threads
        const float v = sh.wtop[lane];
        int above = 0;
        for (int f = 0; f < 32; ++f) {
            const float w = sh.wtop[f];
            above += (w > v) || (w == v && f < lane);
        }
        const unsigned is_k = __ballot_sync(0xffffffffu, above == K - 1);
        tau0 = __shfl_sync(0xffffffffu, v, __ffs(is_k) - 1);
    }
    // pass 2 (the slice is in L2 now): candidates z >= tau0
    auto cand = [&](float x) {
        if (x >= tau0 && x != -INFINITY) {
            const int at = atomicAdd(&sh.ncand, 1);
            if (at < 64) sh.cand[at] = x;
        }
    };
    if (cmax != -INFINITY) {
        for (int i = tid; i < n4; i += 4 * kThreads) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = i + u * kThreads < n4 ? z4[i + u * kThreads] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                cand(v[u].x);
                cand(v[u].y);
                cand(v[u].z);
                cand(v[u].w);
            }
        }
        for (int i = 4 * n4 + tid; i < cnt; i += kThreads) cand(z[i]);
    }
    __syncthreads();
    const int ncand = sh.ncand;
    if (ncand <= 64) {
        if (warp == 0) {
            float x = lane < ncand ? sh.cand[lane] : -INFINITY;
            float y = lane + 32 < ncand ? sh.cand[lane + 32] : -INFINITY;
            warp_sort64_desc(x, y);
            if (lane < K) sh.topk[lane] = x;  // -inf pads a slice shorter than k
            if (lane + 32 < K) sh.topk[lane + 32] = y;
        }
    } else {
        // exact fallback (many equal logits): radix search for the k-th largest key of the slice (four 8-bit
        // digits, counts in shared memory), then the values above it, sorted, then copies of it
        if (tid == 0) {
            sh.fb_prefix = 0;
            sh.fb_pmask = 0;
            sh.fb_above = 0;
            sh.fb_remaining = K;
        }
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = tid; i < 256; i += kThreads) sh.hist[i] = 0;
            __syncthreads();
            const uint32_t prefix = sh.fb_prefix, pmask = sh.fb_pmask;
            for (int i = tid; i < cnt; i += kThreads) {
                const float x = z[i];
                if (x == -INFINITY || !is_finite(x)) continue;
                const uint32_t k = float_key(x);
                if ((k & pmask) == prefix) atomicAdd(&sh.hist[(k >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid == 0) {
                int run = 0;
                for (int b = 255; b >= 0; --b) {
                    const int c = (int)sh.hist[b];
                    if (run + c >= sh.fb_remaining) {
                        sh.fb_above += run;
                        sh.fb_remaining -= run;
                        sh.fb_prefix |= (uint32_t)b << shift;
                        sh.fb_pmask |= 255u << shift;
                        break;
                    }
                    run += c;
                }
            }
            __syncthreads();
        }
        const uint32_t T = sh.fb_prefix;
        const int above = sh.fb_above;  // values strictly greater than T: fewer than k
        if (tid == 0) sh.ncand = 0;
        __syncthreads();
        for (int i = tid; i < cnt; i += kThreads) {
            const float x = z[i];
            if (x != -INFINITY && is_finite(x) && float_key(x) > T) sh.cand[atomicAdd(&sh.ncand, 1)] = x;
        }
        __syncthreads();
        if (warp == 0) {
            float x = lane < above ? sh.cand[lane] : -INFINITY;
            float y = lane + 32 < above ? sh.cand[lane + 32] : -INFINITY;
            warp_sort64_desc(x, y);
            const float tv = key_float(T);
            if (lane < K) sh.topk[lane] = lane < above ? x : tv;
            if (lane + 32 < K) sh.topk[lane + 32] = lane + 32 < above ? y : tv;
        }
    }
    if (tid == 0) {
        sh.cmax = cmax;
        sh.csum = csum;
        sh.nbad = bad;
    }
    cluster.sync();
    if (rank == 0) {
        // merge the cluster: LSE from the (max, sum) pairs; the sum of the k largest from the sorted lists,
        // gathered into the exact fallback's histogram (free again by now) when they fit, else read in place
        float *allv = reinterpret_cast<float *>(sh.hist);
        const bool gathered = K * kCluster <= 256;
        __shared__ float pm[kCluster];
        __shared__ double ps[kCluster];
        __shared__ int anybad;
        if (tid < kCluster) {
            ConfShared *peer = cluster.map_shared_rank(&sh, tid);
            pm[tid] = peer->cmax;
            ps[tid] = peer->csum;
            if (tid == 0) anybad = 0;
        }
        if (gathered)
            for (int e = tid; e < kCluster * K; e += kThreads) allv[e] = cluster.map_shared_rank(&sh, e / K)->topk[e % K];
        __syncthreads();
        if (tid < kCluster && cluster.map_shared_rank(&sh, tid)->nbad) atomicOr(&anybad, 1);
        if (warp == 0) {
            // k steps of taking the largest head among the kCluster lists (lane r holds list r's head)
            int head = 0;
            double topsum = 0.0;
            for (int t = 0; t < K; ++t) {
                const float hv = (lane < kCluster && head < K)
                                     ? (gathered ? allv[lane * K + head] : cluster.map_shared_rank(&sh, lane)->topk[head])
                                     : -INFINITY;
                float best = hv;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
                if (best == -INFINITY) break;  // fewer than k values in the whole row
                const unsigned who = __ballot_sync(0xffffffffu, lane < kCluster && hv == best);
                if (lane == __ffs(who) - 1) ++head;
                topsum += (double)best;
            }
            __syncwarp();
            if (lane == 0) {
                float M = -INFINITY;
                for (int q = 0; q < kCluster; ++q) M = fmaxf(M, pm[q]);
                double S = 0.0;
                for (int q = 0; q < kCluster; ++q)
                    if (pm[q] != -INFINITY) S += ps[q] * exp((double)pm[q] - (double)M);
                const double lse = (double)M + log(S);
                const int kk = min(K, a.vocab);
                const double c = lse - topsum / kk;
                if (anybad) report(a.status, KVC_DEV_NONFINITE, seq);
                a.hist[(int64_t)seq * a.hist_len + (a.window - 1) + step] = (float)c;
                if (a.conf_out) a.conf_out[(int64_t)seq * a.steps + step] = (float)c;
            }
        }
    }
    cluster.sync();
}

struct UpdArgs {
    kvc_ratchet_seq_state *st;
    float *hist;
    int32_t *budget;
    int32_t num_seqs, steps, hist_len;
    kvc_ratchet_params p;
    int32_t staged;     // the call's history (window - 1 + steps floats per warp) fits shared memory
};

// One warp per sequence: the lanes share each window's minimum and the history shift; lane 0 keeps
// the least-squares sums and takes the decision.  The warp first copies the sequence's history into shared
// memory with all its loads in flight, so the windows' minima read shared memory instead of waiting on a
// global load per window (calls whose history does not fit read global memory).
__global__ void ratchet_update_kernel(UpdArgs a) {
    extern __shared__ float hs_all[];   // [warps of the CTA][window - 1 + steps]
    const int lane = threadIdx.x & 31;
    const int seq = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (seq >= a.num_seqs) return;
    kvc_ratchet_seq_state s = a.st[seq];
    float *h = a.hist + (int64_t)seq * a.hist_len;
    const int W = a.p.window, R = a.p.stride;
    const int nh = W - 1 + a.steps;     // the entries this call reads
    const float *hs = h;
    if (a.staged) {
        float *st = hs_all + (size_t)(threadIdx.x >> 5) * nh;
        for (int k = lane; k < nh; k += 32) st[k] = h[k];
        __syncwarp();
        hs = st;
    }
    const int64_t t0 = s.steps_seen, t1 = t0 + a.steps;
    const int64_t base = t0 - (W - 1);  // global step held by h[0]
    int64_t j = s.next_window;
    for (; (int64_t)R * j + W <= t1; ++j) {
        const int64_t ws = (int64_t)R * j;
        float y = INFINITY;
        for (int64_t t = ws + lane; t < ws + W; t += 32) y = fminf(y, hs[t - base]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) y = fminf(y, __shfl_xor_sync(0xffffffffu, y, o));
        if (ws >= s.last_expand_step) {
            const double x = (double)j, yy = (double)y;
            s.fit_n += 1.0;
            s.fit_sx += x;
            s.fit_sy += yy;
            s.fit_sxy += x * yy;
            s.fit_sxx += x * x;
        }
    }
    s.next_window = j;
    s.last_points = (int32_t)s.fit_n;
    s.last_slope = __longlong_as_double(0x7ff8000000000000LL);  // NaN: no evaluation
    if (s.fit_n >= (double)a.p.min_points && s.fit_n >= 2.0) {
        const double n = s.fit_n;
        const double slope = (n * s.fit_sxy - s.fit_sx * s.fit_sy) / (n * s.fit_sxx - s.fit_sx * s.fit_sx);
        s.last_slope = slope;
        if (slope < 0.0) {
            const int64_t nb = (int64_t)s.budget * a.p.grow_num / a.p.grow_den;
            s.budget = (int32_t)(nb < a.p.cap ? nb : a.p.cap);
            s.expansions += 1;
            s.last_expand_step = t1;
            s.fit_n = s.fit_sx = s.fit_sy = s.fit_sxy = s.fit_sxx = 0.0;
        }
    }
    // keep the last window-1 confidences for windows that straddle the next call; chunks ascend and each
    // reads before it writes, so the overlapping forward copy is safe
    for (int k0 = 0; k0 < W - 1; k0 += 32) {
        const int k = k0 + lane;
        const float v = k < W - 1 ? hs[k + a.steps] : 0.f;
        __syncwarp();
        if (k < W - 1) h[k] = v;
        __syncwarp();
    }
    s.steps_seen = t1;
    if (lane == 0) {
        a.st[seq] = s;
        a.budget[seq] = s.budget;
    }
}

__global__ void ratchet_init_kernel(kvc_ratchet_seq_state *st, float *hist, int32_t *budget, int32_t num_seqs,
                                    int32_t hist_len, int32_t init_budget) {
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (tid < num_seqs) {
        kvc_ratchet_seq_state s;
        s.steps_seen = 0;
        s.last_expand_step = 0;
        s.next_window = 0;
        s.fit_n = s.fit_sx = s.fit_sy = s.fit_sxy = s.fit_sxx = 0.0;
        s.last_slope = __longlong_as_double(0x7ff8000000000000LL);
        s.budget = init_budget;
        s.expansions = 0;
        s.last_points = 0;
        s.reserved = 0;
        st[tid] = s;
        if (budget) budget[tid] = init_budget;
    }
    for (int64_t e = tid; e < (int64_t)num_seqs * hist_len; e += (int64_t)gridDim.x * blockDim.x) hist[e] = 0.f;
}

}  // namespace

size_t ratchet_state_bytes(int32_t num_seqs, const kvc_ratchet_params &p) {
    RatchetLayout l = layout_of(num_seqs, p);
    return l.state_bytes + align16((size_t)num_seqs * l.hist_len * sizeof(float));
}

cudaError_t launch_ratchet_init(void *state, int32_t *budget, int32_t num_seqs, const kvc_ratchet_params &p,
                                cudaStream_t stream) {
    RatchetLayout l = layout_of(num_seqs, p);
    auto *st = static_cast<kvc_ratchet_seq_state *>(state);
    float *hist = reinterpret_cast<float *>(static_cast<char *>(state) + l.state_bytes);
    const int64_t work = std::max<int64_t>(num_seqs, (int64_t)num_seqs * l.hist_len);
    const int blocks = (int)std::min<int64_t>(1024, (work + 255) / 256);
    ratchet_init_kernel<<<std::max(blocks, 1), 256, 0, stream>>>(st, hist, budget, num_seqs, l.hist_len,
                                                                  p.init_budget);
    return cudaGetLastError();
}

cudaError_t launch_ratchet(const float *logits, int32_t num_seqs, int32_t steps, int32_t vocab, void *state,
                           int32_t *budget, float *conf_out, const kvc_ratchet_params &p, int32_t *status,
                           cudaStream_t stream) {
    RatchetLayout l = layout_of(num_seqs, p);
    auto *st = static_cast<kvc_ratchet_seq_state *>(state);
    float *hist = reinterpret_cast<float *>(static_cast<char *>(state) + l.state_bytes);
    if (steps > 0) {
        const int chunk = ((vocab + kCluster - 1) / kCluster + 3) / 4 * 4;  // whole 16-byte units per slice
        const int vec = (vocab % 4 == 0) && ((reinterpret_cast<uintptr_t>(logits) & 15) == 0);
        ConfArgs a{logits, steps, vocab, chunk, p.top_k, vec, hist, l.hist_len, p.window, conf_out, status};
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kCluster, (unsigned)steps, (unsigned)num_seqs);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, confidence_kernel, a);
        if (e != cudaSuccess) return e;
    }
    UpdArgs u{st, hist, budget, num_seqs, steps, l.hist_len, p};
    const size_t upd_smem = (size_t)4 * (p.window - 1 + steps) * sizeof(float);
    u.staged = upd_smem <= 48 * 1024;
    ratchet_update_kernel<<<(num_seqs + 3) / 4, 128, u.staged ? upd_smem : 0, stream>>>(u);
    return cudaGetLastError();
}


}  // namespace kvc
