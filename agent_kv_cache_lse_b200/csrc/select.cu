// Top-budget selection; a cluster of C CTAs per row (C = 1..8), each owning a slice.
//
// Eviction keeps the top-`budget` entries of each (sequence, layer, KV head) row by
// their LRFU value, ties broken by the lower token position, then the lower slot
// ("ActKV Dissected", Summary: LRFU eviction policy; the budget is per trajectory).
// Labels selected by protect_label_mask are always kept and use up budget first.
//
// Cluster-wide radix search over order-preserving fp32 keys (four 8-bit digits), then
// over position keys among the entries tied at the threshold; equal (value, position)
// pairs are settled by slot order with a cluster-wide ordered scan.

#include "rowsteps.cuh"

namespace kvc {
namespace {

__global__ void __launch_bounds__(kRowThreads, 1) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RowCtx rc = row_ctx();
    select_row(a, rc, smem_raw);
}

}  // namespace

cudaError_t launch_select(const CacheView &c, const float *crf, const int32_t *budget, uint32_t protect,
                          uint8_t *keep, int32_t *kept, int32_t *status, cudaStream_t stream) {
    const int sms = device_sms();
    const int C = row_cluster_size(c.rows, sms);
    const int per = (int)((c.max_slots + C - 1) / C);
    const int cap = per < 40960 ? per : 0;
    const size_t smem = sizeof(RowShared) + (size_t)cap * 4;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)select_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    SelectArgs a{c, crf, budget, protect, keep, kept, status, cap};
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
    return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace kvc
