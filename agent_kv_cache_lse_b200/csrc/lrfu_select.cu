// Hit gate + LRFU update and top-budget selection in one launch.
//
// The same two per-row bodies as lrfu_kernel and select_kernel ("ActKV Dissected",
// Component 1 and Summary), run back to back by one cluster per row: the selection starts
// on the LRFU values this cluster has just written, with no second launch and no second
// cold read of the row.  Results are those of the two separate calls in sequence.
#include "rowsteps.cuh"

namespace kvc {
namespace {

__global__ void __launch_bounds__(kRowThreads, 1) lrfu_select_kernel(LrfuArgs la, SelectArgs sa) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RowCtx rc = row_ctx();
    lrfu_row(la, rc, smem_raw);
    select_row(sa, rc, smem_raw);
}

}  // namespace

cudaError_t launch_lrfu_select(const CacheView &c, const float *scores, float *crf, float decay, float hit_mass,
                               bool binary, const int32_t *budget, uint32_t protect, uint8_t *keep, int32_t *kept,
                               int32_t *status, cudaStream_t stream) {
    const int sms = device_sms();
    int C = row_cluster_size(c.rows, sms);
    while (C < 8 && (c.max_slots + C - 1) / C > 65536) C <<= 1;  // the mass chunks need slices of at most 2^16
    if ((c.max_slots + C - 1) / C > 65536) return cudaErrorInvalidValue;
    const int per = (int)((c.max_slots + C - 1) / C);
    const int cap = per < 40960 ? per : 0;
    const int wcap = cap > 0 && per <= 12288 ? per : 0;
    const size_t smem = sizeof(RowShared) + (((size_t)cap * 4 + 15) & ~(size_t)15) + (size_t)wcap * 8;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)lrfu_select_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    LrfuArgs la{c, scores, crf, decay, hit_mass, binary ? 1 : 0, status, cap, wcap};
    SelectArgs sa{c, crf, budget, protect, keep, kept, status, cap};
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
    return cudaLaunchKernelEx(&cfg, lrfu_select_kernel, la, sa);
}

}  // namespace kvc
