// Step-aware ranking scores: token saliency blended with the utility of the entry's reasoning step.
//
// "StepKV: Step-Aware KV Cache Compression for LLM Agents" (abstract): entries are tied to the
// step that generated them, each step gets a utility from trajectory signals, and that utility is
// combined with token-level saliency into the scores that rank the prunable tokens under the
// budget.  The page gives no formulas; the ones computed here, per row (sequence, layer, KV head):
//   step(i)  = the last step of the sequence whose start position is at or before slot_pos[i]
//              (steps begin at 0 and where reasoning segments begin; the caller passes the
//              starts, so the step follows the entry through compaction);
//   U_k      = the mean score of the row's entries of step k;
//   out[i]   = (1 - beta) * s[i] + beta * U_step(i).
// The output feeds the same top-budget selection as the LRFU values.
//
// One CTA per row.  Rows of up to 34,816 slots keep their scores in registers (1,024 threads x 34) and
// their step ids in shared memory, so scores and positions are read once; a position's step comes from a
// table of the step at every 2^sh-th position (advanced past any start inside the bucket) instead of a
// binary search.  Longer rows take three passes over global memory.  Pass 1 finds max |s| of the row, which fixes a power-of-two scale; pass 2
// adds every score, rounded to a 64-bit fixed-point integer at that scale, into its step's sum in
// shared memory (integer adds, so the sums do not depend on the order of the atomics; a warp whose
// lanes share a step adds once); pass 3 writes the blend.  The fixed point carries each score to
// within max|s| * 2^-39, far inside fp32 rounding of the blend.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 512;

struct StepArgs {
    CacheView c;
    const float *scores;
    const int32_t *step_start;  // [num_seqs][max_steps]
    const int32_t *num_steps;   // [num_seqs]
    int32_t max_steps;
    float beta;
    float *out;
    int32_t *status;
};

// Step tables up to this size get one copy of the step sums per warp: a warp's adds then never wait on
// another warp's adds to the same step (neighbouring slots share steps, so all warps of a CTA would).
constexpr int kPrivSteps = 64;

// The exact sum over the warp of 64-bit fixed-point values |x| <= 2^39, from two 32-bit reductions:
// x = hi * 2^20 + lo with |hi| <= 2^19 and 0 <= lo < 2^20, so neither 32-lane sum overflows.
__device__ __forceinline__ long long warp_sum_fixed(long long x) {
    const int hs = __reduce_add_sync(0xffffffffu, (int)(x >> 20));
    const unsigned ls = __reduce_add_sync(0xffffffffu, (unsigned)(x & 0xFFFFF));
    return ((long long)hs << 20) + (long long)ls;
}

// adds one warp's (sum, count) of step k: into the warp's own copy when there are copies
__device__ __forceinline__ void add_step(int64_t *sum, int32_t *cnt, int64_t *wsum, int32_t *wcnt, int stride,
                                         int warp, int k, long long t, int c) {
    if (wsum) {
        atomicAdd(reinterpret_cast<unsigned long long *>(&wsum[warp * stride + k]), (unsigned long long)t);
        atomicAdd(&wcnt[warp * stride + k], c);
    } else {
        atomicAdd(reinterpret_cast<unsigned long long *>(&sum[k]), (unsigned long long)t);
        atomicAdd(&cnt[k], c);
    }
}

__device__ __forceinline__ int step_of(const int32_t *starts, int ns, int32_t pos) {
    int lo = 0, hi = ns;  // the answer is in [lo, hi): starts[lo] <= pos (starts[0] = 0 <= pos for pos >= 0)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (starts[mid] <= pos) lo = mid;
        else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kThreads) step_scores_kernel(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int row = blockIdx.x;
    const CacheView &c = a.c;
    const int seq = row / (c.num_layers * c.num_kv_heads);
    int64_t *sum = reinterpret_cast<int64_t *>(smem);                    // [max_steps]
    int32_t *cnt = reinterpret_cast<int32_t *>(sum + a.max_steps);        // [max_steps]
    int32_t *starts = cnt + a.max_steps;                                  // [max_steps]
    const bool priv = a.max_steps <= kPrivSteps;
    int64_t *wsum = priv ? sum + 2 * a.max_steps : nullptr;               // [warps][max_steps] per-warp copies
    int32_t *wcnt = priv ? reinterpret_cast<int32_t *>(wsum + (kThreads / 32) * a.max_steps) : nullptr;
    __shared__ float red[kThreads / 32];
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int n = c.row_len[row];
    const int ns = a.num_steps[seq];
    if (tid == 0) bad = 0;
    __syncthreads();
    if (ns < 1 || ns > a.max_steps) {
        if (tid == 0) report(a.status, KVC_DEV_BAD_STEPS, row);
        return;
    }
    if (n < 0 || n > c.max_slots) {
        if (tid == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const int32_t *st = a.step_start + (int64_t)seq * a.max_steps;
    for (int k = tid; k < ns; k += kThreads) {
        const int32_t v = st[k];
        starts[k] = v;
        sum[k] = 0;
        cnt[k] = 0;
        if ((k == 0 && v != 0) || (k > 0 && v <= st[k - 1])) bad = 1;
    }
    if (priv)
        for (int e = tid; e < (kThreads / 32) * a.max_steps; e += kThreads) {
            wsum[e] = 0;
            wcnt[e] = 0;
        }
    const float *s = a.scores + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    // pass 1: max |s|
    float mx = 0.f;
    for (int i = tid; i < n; i += kThreads) mx = fmaxf(mx, fabsf(s[i]));
    mx = block_max(mx, red);
    if (bad || !is_finite(mx)) {
        if (tid == 0) report(a.status, bad ? KVC_DEV_BAD_STEPS : KVC_DEV_NONFINITE, row);
        return;
    }
    // scale = 2^(39 - E) with max|s| < 2^E: every term below 2^39 in magnitude, any 2^24 of them below 2^63
    int e = 0;
    if (mx > 0.f) frexpf(mx, &e);
    const double scale = ldexp(1.0, 39 - e);
    // pass 2: fixed-point step sums and counts
    for (int i0 = 0; i0 < n; i0 += kThreads) {
        const int i = i0 + tid;
        const bool in = i < n;
        int k = 0;
        long long qv = 0;
        if (in) {
            const int32_t p = pos[i];
            k = p < 0 ? -1 : step_of(starts, ns, p);
            qv = __double2ll_rn((double)s[i] * scale);
        }
        if (in && k < 0) atomicExch(&bad, 1);
        const bool valid = in && k >= 0;
        const unsigned vm = __ballot_sync(0xffffffffu, valid);
        const int k0 = __shfl_sync(0xffffffffu, k, __ffs(vm | 1u) - 1);
        if (vm == 0xffffffffu && __all_sync(0xffffffffu, k == k0)) {
            const long long t = warp_sum_fixed(qv);
            if (lane == 0) add_step(sum, cnt, wsum, wcnt, a.max_steps, warp, k0, t, 32);
        } else if (valid) {
            add_step(sum, cnt, wsum, wcnt, a.max_steps, warp, k, qv, 1);
        }
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) report(a.status, KVC_DEV_BAD_STEPS, row);
        return;
    }
    // step utilities, in place of the sums (as doubles)
    double *u = reinterpret_cast<double *>(sum);
    for (int k = tid; k < ns; k += kThreads) {
        long long t = sum[k];
        int cn = cnt[k];
        if (priv)
            for (int w = 0; w < kThreads / 32; ++w) {
                t += wsum[w * a.max_steps + k];
                cn += wcnt[w * a.max_steps + k];
            }
        u[k] = cn > 0 ? (double)t / (scale * (double)cn) : 0.0;
    }
    __syncthreads();
    // pass 3: the blend
    float *o = a.out + (int64_t)row * c.max_slots;
    const float w = 1.f - a.beta;
    for (int i = tid; i < n; i += kThreads) {
        const float uk = (float)u[step_of(starts, ns, pos[i])];
        o[i] = fmaf(a.beta, uk, w * s[i]);
    }
}

// Rows of at most kRegThreads * kRegSlots slots: each thread keeps its slots' scores in registers and their
// step ids in shared memory, so the row's scores and positions are read from HBM once.
constexpr int kRegThreads = 1024;
constexpr int kRegSlots = 34;  // 34,816 slots: the 33K-token rows of the workloads

__global__ void __launch_bounds__(kRegThreads, 1) step_scores_reg_kernel(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int row = blockIdx.x;
    const CacheView &c = a.c;
    const int seq = row / (c.num_layers * c.num_kv_heads);
    int64_t *sum = reinterpret_cast<int64_t *>(smem);                    // [max_steps]
    int32_t *cnt = reinterpret_cast<int32_t *>(sum + a.max_steps);        // [max_steps]
    int32_t *starts = cnt + a.max_steps;                                  // [max_steps]
    uint16_t *sid = reinterpret_cast<uint16_t *>(starts + a.max_steps);  // [kRegThreads * kRegSlots] step ids
    const bool priv = a.max_steps <= kPrivSteps;
    // [warps][max_steps] per-warp copies of the sums and counts, after the step ids (8-byte aligned: the ids
    // take 2 * kRegThreads * kRegSlots bytes and what precedes them 16 * max_steps)
    int64_t *wsum = priv ? reinterpret_cast<int64_t *>(sid + kRegThreads * kRegSlots) : nullptr;
    int32_t *wcnt = priv ? reinterpret_cast<int32_t *>(wsum + (kRegThreads / 32) * a.max_steps) : nullptr;
    __shared__ float red[kRegThreads / 32];
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int n = c.row_len[row];
    const int ns = a.num_steps[seq];
    if (tid == 0) bad = 0;
    __syncthreads();
    if (ns < 1 || ns > a.max_steps) {
        if (tid == 0) report(a.status, KVC_DEV_BAD_STEPS, row);
        return;
    }
    if (n < 0 || n > c.max_slots) {
        if (tid == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const int32_t *st = a.step_start + (int64_t)seq * a.max_steps;
    for (int k = tid; k < ns; k += kRegThreads) {
        const int32_t v = st[k];
        starts[k] = v;
        sum[k] = 0;
        cnt[k] = 0;
        if ((k == 0 && v != 0) || (k > 0 && v <= st[k - 1])) bad = 1;
    }
    if (priv)
        for (int e = tid; e < (kRegThreads / 32) * a.max_steps; e += kRegThreads) {
            wsum[e] = 0;
            wcnt[e] = 0;
        }
    const float *s = a.scores + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    float v[kRegSlots];
#pragma unroll
    for (int j = 0; j < kRegSlots; ++j) {  // the row's scores, all loads in flight together
        const int i = tid + j * kRegThreads;
        v[j] = i < n ? s[i] : 0.f;
    }
    __syncthreads();  // the step table is in place
    // the step of every 2^sh-th position below the last start, so that a position's step is the bucket's step
    // advanced past the (rare) starts inside the bucket
    __shared__ uint16_t tbl[1024];
    const int32_t last = starts[ns - 1];
    int sh = 0;
    while ((last >> sh) >= 1024) ++sh;
    const int nb = (last >> sh) + 1;
    for (int b = tid; b < nb; b += kRegThreads) tbl[b] = (uint16_t)step_of(starts, ns, b << sh);
    __syncthreads();
    constexpr int kPart = 8;
#pragma unroll
    for (int h = 0; h < (kRegSlots + kPart - 1) / kPart; ++h) {  // positions in parts, to stay within the registers
        int32_t p[kPart];
#pragma unroll
        for (int j = 0; j < kPart; ++j) {
            const int i = tid + (h * kPart + j) * kRegThreads;
            p[j] = (h * kPart + j < kRegSlots && i < n) ? pos[i] : 0;
        }
#pragma unroll
        for (int j = 0; j < kPart; ++j) {
            const int i = tid + (h * kPart + j) * kRegThreads;
            if (h * kPart + j < kRegSlots && i < n) {
                if (p[j] < 0) bad = 1;
                else {
                    int k = ns - 1;
                    if (p[j] < last) {
                        k = tbl[p[j] >> sh];
                        while (starts[k + 1] <= p[j]) ++k;  // k + 1 < ns: p < last = starts[ns - 1]
                    }
                    sid[i] = (uint16_t)k;
                }
            }
        }
    }
    float mx = 0.f;
#pragma unroll
    for (int j = 0; j < kRegSlots; ++j) mx = fmaxf(mx, fabsf(v[j]));
    mx = block_max(mx, red);
    if (bad || !is_finite(mx)) {
        if (tid == 0) report(a.status, bad ? KVC_DEV_BAD_STEPS : KVC_DEV_NONFINITE, row);
        return;
    }
    int e = 0;
    if (mx > 0.f) frexpf(mx, &e);
    const double scale = ldexp(1.0, 39 - e);
#pragma unroll
    for (int j = 0; j < kRegSlots; ++j) {
        const int i = tid + j * kRegThreads;
        if (j * kRegThreads >= n) break;  // block-uniform
        const bool in = i < n;
        const int k = in ? sid[i] : 0;
        const long long qv = in ? __double2ll_rn((double)v[j] * scale) : 0;
        const unsigned vm = __ballot_sync(0xffffffffu, in);
        const int k0 = __shfl_sync(0xffffffffu, k, 0);
        if (vm == 0xffffffffu && __all_sync(0xffffffffu, k == k0)) {
            const long long t = warp_sum_fixed(qv);
            if (lane == 0) add_step(sum, cnt, wsum, wcnt, a.max_steps, warp, k0, t, 32);
        } else if (in) {
            add_step(sum, cnt, wsum, wcnt, a.max_steps, warp, k, qv, 1);
        }
    }
    __syncthreads();
    double *u = reinterpret_cast<double *>(sum);
    for (int k = tid; k < ns; k += kRegThreads) {
        long long t = sum[k];
        int cn = cnt[k];
        if (priv)
            for (int w = 0; w < kRegThreads / 32; ++w) {
                t += wsum[w * a.max_steps + k];
                cn += wcnt[w * a.max_steps + k];
            }
        u[k] = cn > 0 ? (double)t / (scale * (double)cn) : 0.0;
        reinterpret_cast<float *>(cnt)[k] = (float)u[k];  // the blend's fp32 utility, over the count just read
    }
    __syncthreads();
    const float *uf = reinterpret_cast<const float *>(cnt);
    float *o = a.out + (int64_t)row * c.max_slots;
    const float w = 1.f - a.beta;
#pragma unroll
    for (int j = 0; j < kRegSlots; ++j) {
        const int i = tid + j * kRegThreads;
        if (i < n) o[i] = fmaf(a.beta, uf[sid[i]], w * v[j]);
    }
}

}  // namespace

cudaError_t launch_step_scores(const CacheView &c, const float *scores, const int32_t *step_start,
                               const int32_t *num_steps, int32_t max_steps, float beta, float *out, int32_t *status,
                               cudaStream_t stream) {
    if (c.max_slots <= (int64_t)kRegThreads * kRegSlots && max_steps <= 65536) {
        const size_t smem = (size_t)max_steps * (8 + 4 + 4) + (size_t)kRegThreads * kRegSlots * 2 +
                            (max_steps <= kPrivSteps ? (size_t)(kRegThreads / 32) * max_steps * (8 + 4) : 0);
        static int smem_set[kMaxDevices];
        cudaError_t e = dyn_smem_at_least((const void *)step_scores_reg_kernel, smem, smem_set);
        if (e != cudaSuccess) return e;
        step_scores_reg_kernel<<<c.rows, kRegThreads, smem, stream>>>(
            StepArgs{c, scores, step_start, num_steps, max_steps, beta, out, status});
        return cudaGetLastError();
    }
    const size_t smem = (size_t)max_steps * (8 + 4 + 4) +
                        (max_steps <= kPrivSteps ? (size_t)(kThreads / 32) * max_steps * (8 + 4) : 0);
    if (smem > 48 * 1024) {
        static int smem_set[kMaxDevices];
        cudaError_t e = dyn_smem_at_least((const void *)step_scores_kernel, smem, smem_set);
        if (e != cudaSuccess) return e;
    }
    step_scores_kernel<<<c.rows, kThreads, smem, stream>>>(
        StepArgs{c, scores, step_start, num_steps, max_steps, beta, out, status});
    return cudaGetLastError();
}

}  // namespace kvc
