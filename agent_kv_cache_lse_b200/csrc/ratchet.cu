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
//   logits.  Each CTA stages its slice of the vocabulary in shared memory, reduces
//   its (max, sum of exp) and its exact top-k list, and the leader CTA merges the
//   cluster's partials through distributed shared memory into c_t.  The slice arrives
//   by bulk (TMA) copies when the row is 16-byte aligned.  The local top-k takes the
//   k-th largest of the warps' top-2 per-thread maxima as a lower bound, collects the
//   values above it (a few dozen) and sorts them with a warp bitonic network; when
//   more than 64 qualify (many equal logits) it falls back to an exact radix search
//   over the staged slice.
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
constexpr int kThreads = 512;
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
    int32_t bulk;       // rows and slices 16-byte aligned: stage with bulk copies
    float *hist;        // [seqs][hist_len]
    int32_t hist_len, window;
    float *conf_out;    // [seqs][steps] or null
    int32_t *status;
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

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
    RadixShared rs;
    float cand[64];
    float topk[kMaxTopK];
    float wtop[32];      // top-2 per warp of the per-thread maxima
    float red_f[32];
    double red_d[32];
    int red_i[32];
    uint64_t bar;
    float cmax;
    double csum;
    int ncand;
    int nbad;
};

__global__ void __launch_bounds__(kThreads) confidence_kernel(ConfArgs a) {
    extern __shared__ __align__(16) float zs[];
    __shared__ ConfShared sh;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int step = blockIdx.y, seq = blockIdx.z;
    const int K = a.top_k;
    const float *row = a.logits + ((int64_t)seq * a.steps + step) * a.vocab;
    const int lo = min(a.vocab, rank * a.chunk), hi = min(a.vocab, lo + a.chunk);
    const int cnt = hi - lo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // stage the slice in shared memory: one bulk copy when the row slice is 16-byte aligned
    if (tid == 0) {
        sh.ncand = 0;
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&sh.bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const bool bulk = a.bulk && cnt > 0;
    if (bulk) {
        if (tid == 0) {
            const uint32_t bytes = (uint32_t)cnt * 4u;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(&sh.bar)), "r"(bytes)
                         : "memory");
            for (uint32_t off = 0; off < bytes; off += 16384u) {
                const uint32_t sz = min(16384u, bytes - off);
                asm volatile(
                    "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                        smem_addr(zs) + off),
                    "l"(reinterpret_cast<const char *>(row + lo) + off), "r"(sz), "r"(smem_addr(&sh.bar))
                    : "memory");
            }
        }
        // bounded wait for the copy (a second at most)
        uint32_t done = 0;
        long long t0 = clock64();
        while (!done) {
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
                : "=r"(done)
                : "r"(smem_addr(&sh.bar))
                : "memory");
            if (!done && clock64() - t0 > (1ll << 31)) {
                if (tid == 0) report(a.status, KVC_DEV_TIMEOUT, seq);
                break;
            }
        }
    } else {
        for (int i = tid; i < cnt; i += kThreads) zs[i] = row[lo + i];
        __syncthreads();
    }
    // per-thread maximum and finiteness (from shared memory)
    float tmax = -INFINITY;
    int bad = 0;
    for (int i = tid; i < cnt; i += kThreads) {
        const float z = zs[i];
        bad |= !is_finite(z);
        tmax = fmaxf(tmax, z);
    }
    // lower bound tau0 for the slice's k-th largest: the k-th largest of the 32 warp top-2 values
    {
        float m1 = tmax;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        const unsigned who = __ballot_sync(0xffffffffu, tmax == m1);
        float m2 = (lane == __ffs(who) - 1) ? -INFINITY : tmax;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, o));
        if (lane == 0) {
            sh.wtop[2 * warp] = m1;
            sh.wtop[2 * warp + 1] = m2;
        }
    }
    const float cmax = block_max(tmax, sh.red_f);   // also orders the wtop writes
    bad = block_or(bad, sh.red_i);
    float tau0 = -INFINITY;
    if (cnt >= K && K <= 2 * (kThreads / 32)) {
        // every thread ranks the 32 candidates for the bound; identical in all threads
        const float v = sh.wtop[lane];
        int above = 0;
        for (int f = 0; f < 32; ++f) {
            const float w = sh.wtop[f];
            above += (w > v) || (w == v && f < lane);
        }
        const unsigned is_k = __ballot_sync(0xffffffffu, above == K - 1);
        tau0 = __shfl_sync(0xffffffffu, v, __ffs(is_k) - 1);
    }
    // log-sum-exp partial and candidates z >= tau0 (one pass over shared memory)
    float part = 0.f;
    if (cmax != -INFINITY) {
        for (int i = tid; i < cnt; i += kThreads) {
            const float z = zs[i];
            part += exp2f_fast((z - cmax) * 1.4426950408889634f);
            if (z >= tau0) {
                const int at = atomicAdd(&sh.ncand, 1);
                if (at < 64) sh.cand[at] = z;
            }
        }
    }
    const double csum = block_sum<double>((double)part, sh.red_d);  // also orders the candidate writes
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
        // exact fallback (many equal logits): k-th largest key over the staged slice, then values above it
        const RadixResult r = radix_search_desc<false>(
            cnt, (unsigned long long)K, [&](int i) { return float_key(zs[i]); }, [](int) { return 1ull; },
            [](int) { return true; }, sh.rs);
        const float T = key_float(r.key);
        if (tid == 0) sh.ncand = 0;
        __syncthreads();
        for (int i = tid; i < cnt; i += kThreads)
            if (float_key(zs[i]) > r.key) sh.topk[atomicAdd(&sh.ncand, 1)] = zs[i];
        __syncthreads();
        for (int t = (int)r.above + tid; t < K; t += kThreads) sh.topk[t] = T;
    }
    if (tid == 0) {
        sh.cmax = cmax;
        sh.csum = csum;
        sh.nbad = bad;
    }
    cluster.sync();
    if (rank == 0) {
        // merge the cluster: LSE from the partial (max, sum) pairs; global top-k from the local lists
        __shared__ float allv[kCluster * kMaxTopK];
        __shared__ float pm[kCluster];
        __shared__ double ps[kCluster];
        __shared__ int anybad;
        if (tid < kCluster) {
            ConfShared *peer = cluster.map_shared_rank(&sh, tid);
            pm[tid] = peer->cmax;
            ps[tid] = peer->csum;
        }
        if (tid == 0) anybad = 0;
        __syncthreads();
        for (int e = tid; e < kCluster * K; e += kThreads) {
            ConfShared *peer = cluster.map_shared_rank(&sh, e / K);
            allv[e] = peer->topk[e % K];
            if (e % K == 0 && peer->nbad) atomicOr(&anybad, 1);
        }
        __syncthreads();
        double contrib = 0.0;
        for (int e = tid; e < kCluster * K; e += kThreads) {
            const float v = allv[e];
            int above = 0;
            for (int f = 0; f < kCluster * K; ++f) {
                const float w = allv[f];
                above += (w > v) || (w == v && f < e);
            }
            if (above < K && v != -INFINITY) contrib += (double)v;
        }
        const double topsum = block_sum<double>(contrib, sh.red_d);
        if (tid == 0) {
            float M = -INFINITY;
            for (int r = 0; r < kCluster; ++r) M = fmaxf(M, pm[r]);
            double S = 0.0;
            for (int r = 0; r < kCluster; ++r)
                if (pm[r] != -INFINITY) S += ps[r] * exp((double)pm[r] - (double)M);
            const double lse = (double)M + log(S);
            const int kk = min(K, a.vocab);
            const double c = lse - topsum / kk;
            if (anybad) report(a.status, KVC_DEV_NONFINITE, seq);
            a.hist[(int64_t)seq * a.hist_len + (a.window - 1) + step] = (float)c;
            if (a.conf_out) a.conf_out[(int64_t)seq * a.steps + step] = (float)c;
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
};

// One warp per sequence: the lanes share each window's minimum and the history shift; lane 0 keeps
// the least-squares sums and takes the decision.
__global__ void ratchet_update_kernel(UpdArgs a) {
    const int lane = threadIdx.x & 31;
    const int seq = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (seq >= a.num_seqs) return;
    kvc_ratchet_seq_state s = a.st[seq];
    float *h = a.hist + (int64_t)seq * a.hist_len;
    const int W = a.p.window, R = a.p.stride;
    const int64_t t0 = s.steps_seen, t1 = t0 + a.steps;
    const int64_t base = t0 - (W - 1);  // global step held by h[0]
    int64_t j = s.next_window;
    for (; (int64_t)R * j + W <= t1; ++j) {
        const int64_t ws = (int64_t)R * j;
        float y = INFINITY;
        for (int64_t t = ws + lane; t < ws + W; t += 32) y = fminf(y, h[t - base]);
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
        const float v = k < W - 1 ? h[k + a.steps] : 0.f;
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
        const size_t smem = (size_t)chunk * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(confidence_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int bulk = (vocab % 4 == 0) && ((reinterpret_cast<uintptr_t>(logits) & 15) == 0);
        ConfArgs a{logits, steps, vocab, chunk, p.top_k, bulk, hist, l.hist_len, p.window, conf_out, status};
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kCluster, (unsigned)steps, (unsigned)num_seqs);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, confidence_kernel, a);
        if (e != cudaSuccess) return e;
    }
    UpdArgs u{st, hist, budget, num_seqs, steps, l.hist_len, p};
    ratchet_update_kernel<<<(num_seqs + 3) / 4, 128, 0, stream>>>(u);
    return cudaGetLastError();
}

int ratchet_max_top_k() { return kMaxTopK; }
int ratchet_max_vocab() { return 40960 * kCluster; }

}  // namespace kvc
