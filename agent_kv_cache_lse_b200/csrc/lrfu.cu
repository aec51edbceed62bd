// Hit gate + LRFU update; a cluster of C CTAs per row (C = 1..8), each owning a slice.
//
// "ActKV Dissected", Component 1: the entries in the top 90% of the action
// attention are action-critical, and that hit signal replaces LRFU's hit, with
// decay coefficient lambda = 0.5.  "Top 90%" is read as cumulative attention mass:
// the hits are the shortest prefix of the order (score desc, position asc, slot asc)
// whose mass reaches hit_mass of the row's total.
//
// The threshold comes from a cluster-wide radix search whose per-digit masses are
// 64-bit fixed-point integers (scores scaled by a power of two so the row maximum is
// just under 2^48): integer sums make the search independent of summation order, so
// the result is the same run to run.

#include "rowsteps.cuh"

namespace kvc {
namespace {

// At most 96 registers (512 x 96 of the SM's 65,536): the round runs the ratchet's confidence CTAs beside this
// kernel, and the spare registers let two of them share each SM that holds an LRFU CTA.
__global__ void __maxnreg__(96) lrfu_kernel(LrfuArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RowCtx rc = row_ctx();
    lrfu_row(a, rc, smem_raw);
}

}  // namespace

cudaError_t launch_lrfu(const CacheView &c, const float *scores, float *crf, float decay, float hit_mass,
                        bool binary, int32_t *status, cudaStream_t stream) {
    const int sms = device_sms();
    int C = row_cluster_size(c.rows, sms);
    while (C < 8 && (c.max_slots + C - 1) / C > 65536) C <<= 1;  // the mass chunks need slices of at most 2^16
    if ((c.max_slots + C - 1) / C > 65536) return cudaErrorInvalidValue;
    const int per = (int)((c.max_slots + C - 1) / C);
    const int cap = per < 40960 ? per : 0;
    const int wcap = cap > 0 && per <= 12288 ? per : 0;
    const size_t smem = sizeof(RowShared) + (((size_t)cap * 4 + 15) & ~(size_t)15) + (size_t)wcap * 8;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)lrfu_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    LrfuArgs a{c, scores, crf, decay, hit_mass, binary ? 1 : 0, status, cap, wcap};
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
    return cudaLaunchKernelEx(&cfg, lrfu_kernel, a);
}

}  // namespace kvc
