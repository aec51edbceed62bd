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
// their step ids in shared memory, so scores and positions are read once; longer rows take three passes
// over global memory.  Pass 1 finds max |s| of the row, which fixes a power-of-two scale; pass 2
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
    __shared__ float red[kThreads / 32];
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31;

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
            long long t = qv;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            if (lane == 0) {
                atomicAdd(reinterpret_cast<unsigned long long *>(&sum[k0]), (unsigned long long)t);
                atomicAdd(&cnt[k0], 32);
            }
        } else if (valid) {
            atomicAdd(reinterpret_cast<unsigned long long *>(&sum[k]), (unsigned long long)qv);
            atomicAdd(&cnt[k], 1);
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
        const long long t = sum[k];
        u[k] = cnt[k] > 0 ? (double)t / (scale * (double)cnt[k]) : 0.0;
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
    __shared__ float red[kRegThreads / 32];
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31;

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
    const float *s = a.scores + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    float v[kRegSlots];
#pragma unroll
    for (int j = 0; j < kRegSlots; ++j) {  // the row's scores, all loads in flight together
        const int i = tid + j * kRegThreads;
        v[j] = i < n ? s[i] : 0.f;
    }
    __syncthreads();  // the step table is in place
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
                else sid[i] = (uint16_t)step_of(starts, ns, p[j]);
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
            long long t = qv;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            if (lane == 0) {
                atomicAdd(reinterpret_cast<unsigned long long *>(&sum[k0]), (unsigned long long)t);
                atomicAdd(&cnt[k0], 32);
            }
        } else if (in) {
            atomicAdd(reinterpret_cast<unsigned long long *>(&sum[k]), (unsigned long long)qv);
            atomicAdd(&cnt[k], 1);
        }
    }
    __syncthreads();
    double *u = reinterpret_cast<double *>(sum);
    for (int k = tid; k < ns; k += kRegThreads) {
        const long long t = sum[k];
        u[k] = cnt[k] > 0 ? (double)t / (scale * (double)cnt[k]) : 0.0;
    }
    __syncthreads();
    float *o = a.out + (int64_t)row * c.max_slots;
    const float w = 1.f - a.beta;
#pragma unroll
    for (int j = 0; j < kRegSlots; ++j) {
        const int i = tid + j * kRegThreads;
        if (i < n) o[i] = fmaf(a.beta, (float)u[sid[i]], w * v[j]);
    }
}

}  // namespace

cudaError_t launch_step_scores(const CacheView &c, const float *scores, const int32_t *step_start,
                               const int32_t *num_steps, int32_t max_steps, float beta, float *out, int32_t *status,
                               cudaStream_t stream) {
    if (c.max_slots <= (int64_t)kRegThreads * kRegSlots && max_steps <= 65536) {
        const size_t smem = (size_t)max_steps * (8 + 4 + 4) + (size_t)kRegThreads * kRegSlots * 2;
        static int smem_set[kMaxDevices];
        cudaError_t e = dyn_smem_at_least((const void *)step_scores_reg_kernel, smem, smem_set);
        if (e != cudaSuccess) return e;
        step_scores_reg_kernel<<<c.rows, kRegThreads, smem, stream>>>(
            StepArgs{c, scores, step_start, num_steps, max_steps, beta, out, status});
        return cudaGetLastError();
    }
    const size_t smem = (size_t)max_steps * (8 + 4 + 4);
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
