// In-place paged compaction.
//
// "ActKV Dissected", Component 3: after the conflict-free slot plan, surviving
// entries are copied into the holes in one parallel pass, the freed blocks go back
// to the scheduler, and no extra KV buffer is used.
//
// Launch A: one warp per move copies the K and V vectors of the source slot to the
//           destination slot with 16-byte vector loads and stores, plus the slot's
//           position, label and LRFU value.  One extra CTA computes each row's offset
//           in the freed-page list (exclusive scan over rows) into the workspace.
// Launch B: each row's tail pages ceil(m/P) .. ceil(n/P)-1 go to the freed list in
//           row order, their block-table entries become -1, and row_len = m.  It runs
//           after A so no move reads a block-table entry that is being cleared.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 256;

struct CompactArgs {
    CacheView c;
    const int32_t *move_src;
    const int32_t *move_dst;
    const int32_t *num_moves;
    const int32_t *new_len;
    float *crf;
    int32_t *freed;
    int64_t freed_capacity;
    int64_t *num_freed;
    int64_t *row_offsets;  // [rows + 1] workspace
    int32_t *status;
    int row_vec16;         // 16-byte vectors per K (or V) vector
};

__device__ __forceinline__ bool row_ok(const CacheView &c, int n, int m) {
    return n >= 0 && n <= c.max_slots && m >= 0 && m <= n;
}

// A row is compacted only when its lengths and its move count are consistent; any other row (among
// them the rows the planner rejected, num_moves = -1) keeps its pages, block table and row_len.
__device__ __forceinline__ bool row_plan_ok(const CacheView &c, int n, int m, int nm) {
    return row_ok(c, n, m) && nm >= 0 && nm <= m && nm <= n - m;
}

__device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

__device__ void freed_offsets(const CompactArgs &a) {
    __shared__ int red[32];
    __shared__ long long carry_s;
    const CacheView &c = a.c;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int r0 = 0; r0 < c.rows; r0 += blockDim.x) {
        const int r = r0 + threadIdx.x;
        int f = 0;
        if (r < c.rows) {
            const int n = c.row_len[r], m = a.new_len[r];
            if (row_plan_ok(c, n, m, a.num_moves[r])) f = (int)(ceil_div(n, c.page_size) - ceil_div(m, c.page_size));
        }
        int total;
        const int ex = block_exclusive_scan(f, red, &total);
        const long long carry = carry_s;
        if (r < c.rows) a.row_offsets[r] = carry + ex;
        __syncthreads();
        if (threadIdx.x == 0) carry_s = carry + total;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        a.row_offsets[c.rows] = carry_s;
        *a.num_freed = carry_s;
        if (carry_s > a.freed_capacity) report(a.status, KVC_DEV_FREED_OVERFLOW, -1);
    }
}

__global__ void __launch_bounds__(kThreads) compact_moves_kernel(CompactArgs a) {
    const CacheView &c = a.c;
    if ((int)blockIdx.y == c.rows) {
        if (blockIdx.x == 0) freed_offsets(a);
        return;
    }
    const int row = blockIdx.y;
    const int n = c.row_len[row], m = a.new_len[row];
    const int nm = a.num_moves[row];
    if (!row_plan_ok(c, n, m, nm)) {
        // num_moves = -1: the planner rejected the row and has reported why
        if (blockIdx.x == 0 && threadIdx.x == 0 && nm != -1)
            report(a.status, row_ok(c, n, m) ? KVC_DEV_BAD_MOVE : KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
    const int P = c.page_size;
    const int64_t ms = c.max_slots;
    const int32_t *bt = c.block_table + (int64_t)row * c.max_pages_per_row;
    const int nv = a.row_vec16;
    for (int j = blockIdx.x * wpb + (threadIdx.x >> 5); j < nm; j += gridDim.x * wpb) {
        const int s = a.move_src[row * ms + j];
        const int d = a.move_dst[row * ms + j];
        if (s < m || s >= n || d < 0 || d >= m) {
            if (lane == 0) report(a.status, KVC_DEV_BAD_MOVE, row);
            continue;
        }
        const int32_t ps = bt[s / P], pd = bt[d / P];
        if (ps < 0 || ps >= c.num_pages || pd < 0 || pd >= c.num_pages) {
            if (lane == 0) report(a.status, KVC_DEV_BAD_PAGE, row);
            continue;
        }
        const int64_t so = ((int64_t)ps * P + s % P) * nv, dof = ((int64_t)pd * P + d % P) * nv;
        for (int v = lane; v < 2 * nv; v += 32) {
            const bool is_k = v < nv;
            const int e = is_k ? v : v - nv;
            uint4 *pool = static_cast<uint4 *>(const_cast<void *>(is_k ? c.k_pool : c.v_pool));
            pool[dof + e] = pool[so + e];
        }
        if (lane == 0) {
            c.slot_pos[row * ms + d] = c.slot_pos[row * ms + s];
            if (c.slot_label) c.slot_label[row * ms + d] = c.slot_label[row * ms + s];
            if (a.crf) a.crf[row * ms + d] = a.crf[row * ms + s];
        }
    }
}

__global__ void __launch_bounds__(kThreads) compact_free_kernel(CompactArgs a) {
    const CacheView &c = a.c;
    const int row = blockIdx.y;
    const int n = c.row_len[row], m = a.new_len[row];
    if (!row_plan_ok(c, n, m, a.num_moves[row])) return;
    const int64_t first = ceil_div(m, c.page_size), end = ceil_div(n, c.page_size);
    const int64_t base = a.row_offsets[row];
    // all of a row's pages go back, or (when the list is too short) none of them
    const bool fits = base + (end - first) <= a.freed_capacity;
    int32_t *bt = c.block_table + (int64_t)row * c.max_pages_per_row;
    if (fits) {
        for (int64_t p = first + blockIdx.x * blockDim.x + threadIdx.x; p < end; p += (int64_t)gridDim.x * blockDim.x) {
            a.freed[base + (p - first)] = bt[p];
            bt[p] = -1;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) c.row_len[row] = m;
}

}  // namespace

cudaError_t launch_compact(const CacheView &c, const int32_t *move_src, const int32_t *move_dst,
                           const int32_t *num_moves, const int32_t *new_len, float *crf, int32_t *freed,
                           int64_t freed_capacity, int64_t *num_freed, int64_t *row_offsets,
                           int32_t *status, cudaStream_t stream) {
    const int esize = c.dtype == KVC_BF16 ? 2 : 4;
    CompactArgs a{c, move_src, move_dst, num_moves, new_len, crf, freed, freed_capacity, num_freed,
                  row_offsets, status, c.head_dim * esize / 16};
    const int sms = device_sms();
    const int xa = std::max(1, std::min(64, (4 * sms + c.rows - 1) / c.rows));
    compact_moves_kernel<<<dim3(xa, c.rows + 1), kThreads, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int xb = std::max(1, std::min(16, (2 * sms + c.rows - 1) / c.rows));
    compact_free_kernel<<<dim3(xb, c.rows), kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kvc
