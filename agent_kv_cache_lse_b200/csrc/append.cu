// Appending decoded tokens to a compacted cache, taking pages from the free-page stack.
//
// "KV-streams for Efficient Compaction in Agentic Reinforcement Learning" (abstract): instead of flushing the
// cache at a rollout boundary and prefilling the whole context again, the compacted cache is carried
// forward and new tokens stream into it.  After a compaction the rows are dense prefixes [0, row_len) whose
// tail pages went back to the free list; this step writes `count` new tokens per row at slots
// row_len .. row_len + count - 1, mapping a fresh page from the stack wherever a row crosses into a page it
// does not hold.
//
// Launch A (one CTA): per row the pages it needs, an exclusive scan over rows, the total against the stack
//   depth; rows take their pages from the top of the stack in row order (row r's k-th new page is
//   free[depth - total + offset_r + k]) and the depth drops by the total.  If the stack is too shallow the call
//   appends nothing and reports KVC_DEV_FREED_OVERFLOW.
// Launch B (rows x CTAs): block-table entries of the new pages, then one warp per token copies its K and V
//   rows with 16-byte vectors and writes its position, label and zero LRFU value; row_len += count.  Every
//   page a token lands in is computed from the scan (old pages from the block table, new ones from the
//   stack), so no CTA depends on another's writes.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 256;

struct AppendArgs {
    CacheView c;
    const void *k_new, *v_new;
    const int32_t *new_pos;
    int32_t count;
    uint8_t label;
    float *crf;
    int32_t *free_pages;
    int64_t *free_count;
    int64_t *ws;         // [0, rows]: page offsets (ws[rows] = total, ws[rows + 1] = base or -1); [rows + 2, 2 rows + 2): row_len before
    int32_t *status;
    int vec16;           // 16-byte vectors per K (or V) row
};

__device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

__global__ void __launch_bounds__(kThreads) append_plan_kernel(AppendArgs a) {
    __shared__ int red[32];
    __shared__ long long carry_s;
    const CacheView &c = a.c;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int r0 = 0; r0 < c.rows; r0 += blockDim.x) {
        const int r = r0 + threadIdx.x;
        int need = 0;
        if (r < c.rows) {
            const int n = c.row_len[r];
            a.ws[c.rows + 2 + r] = n;
            if (n < 0 || (int64_t)n + a.count > c.max_slots) {
                report(a.status, n < 0 ? KVC_DEV_BAD_LENGTH : KVC_DEV_FREED_OVERFLOW, r);
                a.ws[c.rows + 2 + r] = -1;   // this row is left alone
            } else {
                need = (int)(cdiv((int64_t)n + a.count, c.page_size) - cdiv(n, c.page_size));
            }
        }
        int total;
        const int ex = block_exclusive_scan(need, red, &total);
        const long long carry = carry_s;
        if (r < c.rows) a.ws[r] = carry + ex;
        __syncthreads();
        if (threadIdx.x == 0) carry_s = carry + total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const long long total = carry_s, depth = *a.free_count;
        a.ws[c.rows] = total;
        if (total > depth) {
            report(a.status, KVC_DEV_FREED_OVERFLOW, -1);
            a.ws[c.rows + 1] = -1;           // nothing is appended
        } else {
            a.ws[c.rows + 1] = depth - total;
            *a.free_count = depth - total;
        }
    }
}

__global__ void __launch_bounds__(kThreads) append_write_kernel(AppendArgs a) {
    const CacheView &c = a.c;
    const int row = blockIdx.y;
    const int64_t base = a.ws[c.rows + 1];
    const int n = (int)a.ws[c.rows + 2 + row];
    if (base < 0 || n < 0) return;
    const int P = c.page_size;
    const int64_t first_new = cdiv(n, P), off = a.ws[row];
    int32_t *bt = c.block_table + (int64_t)row * c.max_pages_per_row;
    auto page_of = [&](int64_t lp) -> int32_t {
        return lp < first_new ? bt[lp] : a.free_pages[base + off + (lp - first_new)];
    };
    // block-table entries of the row's new pages (read by nobody in this launch: pages come from the scan)
    const int64_t end = cdiv((int64_t)n + a.count, P);
    for (int64_t lp = first_new + blockIdx.x * blockDim.x + threadIdx.x; lp < end; lp += (int64_t)gridDim.x * blockDim.x)
        bt[lp] = a.free_pages[base + off + (lp - first_new)];
    const int seq = row / (c.num_layers * c.num_kv_heads);
    const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
    const int nv = a.vec16;
    const int64_t ms = c.max_slots;
    for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < a.count; i += gridDim.x * wpb) {
        const int s = n + i;
        const int32_t pg = page_of(s / P);
        if (pg < 0 || pg >= c.num_pages) {
            if (lane == 0) report(a.status, KVC_DEV_BAD_PAGE, row);
            continue;
        }
        const int64_t dof = ((int64_t)pg * P + s % P) * nv, sof = ((int64_t)row * a.count + i) * nv;
        for (int v = lane; v < 2 * nv; v += 32) {
            const bool is_k = v < nv;
            const int e = is_k ? v : v - nv;
            uint4 *pool = static_cast<uint4 *>(const_cast<void *>(is_k ? c.k_pool : c.v_pool));
            const uint4 *src = static_cast<const uint4 *>(is_k ? a.k_new : a.v_new);
            pool[dof + e] = src[sof + e];
        }
        if (lane == 0) {
            c.slot_pos[row * ms + s] = a.new_pos[(int64_t)seq * a.count + i];
            if (c.slot_label) c.slot_label[row * ms + s] = a.label;
            if (a.crf) a.crf[row * ms + s] = 0.f;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) c.row_len[row] = n + a.count;
}

}  // namespace

cudaError_t launch_append(const CacheView &c, const void *k_new, const void *v_new, const int32_t *new_pos,
                          int32_t count, uint8_t label, float *crf, int32_t *free_pages, int64_t *free_count,
                          int64_t *ws, int32_t *status, cudaStream_t stream) {
    const int esize = c.dtype == KVC_BF16 ? 2 : 4;
    AppendArgs a{c, k_new, v_new, new_pos, count, label, crf, free_pages, free_count, ws, status,
                 c.head_dim * esize / 16};
    append_plan_kernel<<<1, kThreads, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    const int per_row_warps = (count + 7) / 8;
    const int xb = std::max(1, std::min(std::max(1, (4 * sms + c.rows - 1) / c.rows), per_row_warps));
    append_write_kernel<<<dim3(xb, c.rows), kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kvc
