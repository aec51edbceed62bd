// Conflict-free slot plan; a cluster of C CTAs per row (C = 1..8), each owning a slice.
//
// "ActKV Dissected", Component 3: naive parallel in-place migration conflicts, so the
// survivors outside the target region are paired one-to-one with the holes inside it
// before a single parallel copy.  The target region is the row's dense prefix [0, m),
// m = number kept: survivor j (ascending, at or after m) fills hole j (ascending,
// before m).  Sources and destinations are disjoint and each destination appears
// once, so the copy pass has no read/write conflicts.
//
// Every thread owns a contiguous run of slots; a CTA scan plus the cluster-wide sums of
// the lower slices give every hole and every survivor its rank, which is its index in
// the move list.
#include "internal.h"
#include "rowcluster.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 512;

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
    __shared__ RowShared sh;
    RowCtx rc = row_ctx();
    const int row = blockIdx.x / rc.nranks;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    const int m = a.kept[row];
    // A rejected row gets num_moves = -1, which the compaction reads as "leave this row as it is".
    if (n < 0 || n > c.max_slots || m < 0 || m > n) {
        if (rc.rank == 0 && threadIdx.x == 0) {
            a.num_moves[row] = -1;
            report(a.status, (n < 0 || n > c.max_slots) ? KVC_DEV_BAD_LENGTH : KVC_DEV_KEPT_MISMATCH, row);
        }
        return;
    }
    const int per = (n + rc.nranks - 1) / rc.nranks;
    const int lo = min(n, rc.rank * per), hi = min(n, lo + per);
    const uint8_t *keep = a.keep + (int64_t)row * c.max_slots;
    const int span = hi - lo;
    const int chunk = (span + blockDim.x - 1) / blockDim.x;
    const int b0 = lo + min(span, (int)threadIdx.x * chunk), b1 = lo + min(span, ((int)threadIdx.x + 1) * chunk);
    int holes = 0, movers = 0;
    for (int i = b0; i < b1; ++i) {
        const int k = keep[i] != 0;
        if (i < m) holes += !k;
        else movers += k;
    }
    int th, tm;
    int hr = block_exclusive_scan(holes, sh.red_i, &th);
    int mr = block_exclusive_scan(movers, sh.red_i, &tm);
    int tot[2], below[2];
    row_sum_int2(rc, sh, holes, movers, tot, below);
    // kept count consistent with the mask  <=>  as many holes before m as survivors after it
    if (tot[0] != tot[1]) {
        if (rc.rank == 0 && threadIdx.x == 0) {
            a.num_moves[row] = -1;
            report(a.status, KVC_DEV_KEPT_MISMATCH, row);
        }
        rc.cl.sync();
        return;
    }
    hr += below[0];
    mr += below[1];
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
    if (rc.rank == 0 && threadIdx.x == 0) a.num_moves[row] = tot[0];
    rc.cl.sync();
}

}  // namespace

cudaError_t launch_plan(const CacheView &c, const uint8_t *keep, const int32_t *kept, int32_t *move_src,
                        int32_t *move_dst, int32_t *num_moves, int32_t *status, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int C = row_cluster_size(c.rows, sms);
    PlanArgs a{c, keep, kept, move_src, move_dst, num_moves, status};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c.rows * C));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, plan_kernel, a);
}

}  // namespace kvc
