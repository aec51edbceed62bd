// Conflict-free slot plan, one CTA per row.
//
// "ActKV Dissected", Component 3: naive parallel in-place migration conflicts, so the
// survivors outside the target region are paired one-to-one with the holes inside it
// before a single parallel copy.  The target region is the row's dense prefix [0, m),
// m = number kept: survivor j (ascending, at or after m) fills hole j (ascending,
// before m).  Sources and destinations are disjoint and each destination appears
// once, so the copy pass has no read/write conflicts.
//
// Each thread owns a contiguous chunk of slots; two CTA exclusive scans give every
// hole and every survivor its rank, which is its index in the move list.
#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 1024;

struct PlanArgs {
    CacheView c;
    const uint8_t *keep;
    const int32_t *kept;
    int32_t *move_src;
    int32_t *move_dst;
    int32_t *num_moves;
    int32_t *status;
};

__global__ void __launch_bounds__(kThreads) plan_kernel(PlanArgs a) {
    __shared__ int red[32];
    const int row = blockIdx.x;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    const int m = a.kept[row];
    if (n < 0 || n > c.max_slots || m < 0 || m > n) {
        if (threadIdx.x == 0) {
            a.num_moves[row] = 0;
            report(a.status, (n < 0 || n > c.max_slots) ? KVC_DEV_BAD_LENGTH : KVC_DEV_KEPT_MISMATCH, row);
        }
        return;
    }
    const uint8_t *keep = a.keep + (int64_t)row * c.max_slots;
    const int chunk = (n + blockDim.x - 1) / blockDim.x;
    const int b0 = min(n, threadIdx.x * chunk), b1 = min(n, b0 + chunk);
    int holes = 0, movers = 0, ones = 0;
    for (int i = b0; i < b1; ++i) {
        const int k = keep[i] != 0;
        ones += k;
        if (i < m) holes += !k;
        else movers += k;
    }
    int th, tm;
    int hr = block_exclusive_scan(holes, red, &th);
    int mr = block_exclusive_scan(movers, red, &tm);
    const int to = block_sum<int>(ones, red);
    if (to != m || th != tm) {
        if (threadIdx.x == 0) {
            a.num_moves[row] = 0;
            report(a.status, KVC_DEV_KEPT_MISMATCH, row);
        }
        return;
    }
    int32_t *src = a.move_src + (int64_t)row * c.max_slots;
    int32_t *dst = a.move_dst + (int64_t)row * c.max_slots;
    for (int i = b0; i < b1; ++i) {
        const int k = keep[i] != 0;
        if (i < m) {
            if (!k) dst[hr++] = i;
        } else if (k) {
            src[mr++] = i;
        }
    }
    if (threadIdx.x == 0) a.num_moves[row] = th;
}

}  // namespace

cudaError_t launch_plan(const CacheView &c, const uint8_t *keep, const int32_t *kept, int32_t *move_src,
                        int32_t *move_dst, int32_t *num_moves, int32_t *status, cudaStream_t stream) {
    PlanArgs a{c, keep, kept, move_src, move_dst, num_moves, status};
    plan_kernel<<<c.rows, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kvc
