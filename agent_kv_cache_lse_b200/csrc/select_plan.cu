// Top-budget selection and the slot plan in one launch.
//
// The same two per-row bodies as select_kernel and plan_kernel ("ActKV Dissected", Summary: LRFU eviction
// under a budget; Component 3: conflict-free slot planning), run back to back by one cluster per row: the plan
// starts on the keep mask and kept count this cluster has just written, with no second launch.  Both bodies
// split the row into the same slices, so each CTA plans the slice it selected; the closing cluster barrier of
// the selection orders its writes before the plan reads them.  Results are those of the two separate calls in
// sequence.
#include "rowsteps.cuh"

namespace kvc {
namespace {

__global__ void __launch_bounds__(kRowThreads, 1) select_plan_kernel(SelectArgs sa, PlanArgs pa) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RowCtx rc = row_ctx();
    select_row(sa, rc, smem_raw);
    plan_row(pa, rc, *reinterpret_cast<RowShared *>(smem_raw));
}

}  // namespace

cudaError_t launch_select_plan(const CacheView &c, const float *crf, const int32_t *budget, uint32_t protect,
                               uint8_t *keep, int32_t *kept, int32_t *move_src, int32_t *move_dst,
                               int32_t *num_moves, int32_t *status, cudaStream_t stream) {
    const int sms = device_sms();
    const int C = row_cluster_size(c.rows, sms);
    const int per = (int)((c.max_slots + C - 1) / C);
    const int cap = per < 40960 ? per : 0;
    const size_t smem = sizeof(RowShared) + (size_t)cap * 4;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)select_plan_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    SelectArgs sa{c, crf, budget, protect, keep, kept, status, cap};
    PlanArgs pa{c, keep, kept, move_src, move_dst, num_moves, status};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c.rows * C));
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, select_plan_kernel, sa, pa);
}

}  // namespace kvc
