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
#include "rowsteps.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 512;

__global__ void __launch_bounds__(kThreads) plan_kernel(PlanArgs a) {
    __shared__ RowShared sh;
    RowCtx rc = row_ctx();
    plan_row(a, rc, sh);
}

}  // namespace

cudaError_t launch_plan(const CacheView &c, const uint8_t *keep, const int32_t *kept, int32_t *move_src,
                        int32_t *move_dst, int32_t *num_moves, int32_t *status, cudaStream_t stream) {
    const int sms = device_sms();
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
