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
#include "internal.h"
#include "rowcluster.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 512;

struct SelectArgs {
    CacheView c;
    const float *crf;
    const int32_t *budget;
    uint32_t protect;
    uint8_t *keep;
    int32_t *kept;
    int32_t *status;
    int slice_cap;
};

__global__ void __launch_bounds__(kThreads, 1) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RowShared &sh = *reinterpret_cast<RowShared *>(smem_raw);
    uint32_t *kc = reinterpret_cast<uint32_t *>(smem_raw + sizeof(RowShared));
    RowCtx rc = row_ctx();
    const int row = blockIdx.x / rc.nranks;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (rc.rank == 0 && threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const int per = (n + rc.nranks - 1) / rc.nranks;
    const int lo = min(n, rc.rank * per), hi = min(n, lo + per);
    const int seq = row / (c.num_layers * c.num_kv_heads);
    const int B = max(a.budget[seq], 0);
    const float *crf = a.crf + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    const uint8_t *lab = c.slot_label ? c.slot_label + (int64_t)row * c.max_slots : nullptr;
    uint8_t *keep = a.keep + (int64_t)row * c.max_slots;
    const bool cached = per <= a.slice_cap;
    const uint32_t protect = lab ? a.protect : 0u;
    auto prot = [&](int i) -> bool { return protect && ((protect >> (lab[i] & 31)) & 1u); };

    int bad = 0, nprot = 0;
    for (int base = lo + threadIdx.x; base < hi; base += 8 * blockDim.x) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // eight independent loads in flight before any is used
            const int i = base + u * blockDim.x;
            v[u] = i < hi ? crf[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * blockDim.x;
            if (i < hi) {
                if (!is_finite(v[u])) bad = 1;
                if (cached) kc[i - lo] = float_key(v[u] == 0.f ? 0.f : v[u]);  // -0.0 ranks as +0.0
                nprot += prot(i) ? 1 : 0;
            }
        }
    }
    // one collective: the protected count and whether any CRF is not finite
    int tot[2], below[2];
    row_sum_int2(rc, sh, nprot, bad, tot, below);
    if (tot[1] != 0) {
        // keep everything on a faulted row: nothing is evicted
        for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) keep[i] = 1;
        if (rc.rank == 0 && threadIdx.x == 0) {
            a.kept[row] = n;
            report(a.status, KVC_DEV_NONFINITE, row);
        }
        rc.cl.sync();
        return;
    }
    nprot = tot[0];
    auto key = [&](int i) -> uint32_t {
        if (cached) return kc[i - lo];
        const float v = crf[i];
        return float_key(v == 0.f ? 0.f : v);
    };
    const int ncand = n - nprot;
    const int room = min(max(B - nprot, 0), ncand);
    const int mode = room >= ncand ? 0 : (room == 0 ? 1 : 2);  // keep all / none / by threshold
    uint32_t T = 0, PK = 0;
    int tie_mode = 0;
    unsigned long long slot_need = 0;
    if (mode == 2) {
        const RadixResult r = row_radix_desc<false>(rc, sh, lo, hi, (unsigned long long)room, key,
                                                    [](int) { return 1ull; }, [&](int i) { return !prot(i); });
        T = r.key;
        const unsigned long long need = room - r.above;
        if (need < r.eq_count) {
            const RadixResult r2 = row_radix_desc<false>(
                rc, sh, lo, hi, need, [&](int i) { return pos_desc_key(pos[i]); }, [](int) { return 1ull; },
                [&](int i) { return !prot(i) && key(i) == T; });
            PK = r2.key;
            tie_mode = 1;
            const unsigned long long need2 = need - r2.above;
            if (need2 < r2.eq_count) {
                tie_mode = 2;
                slot_need = need2;
            }
        }
    }
    auto decide = [&](int i) -> int {
        if (prot(i) || mode == 0) return 1;
        if (mode == 1) return 0;
        const uint32_t k = key(i);
        if (k > T) return 1;
        if (k < T) return 0;
        if (tie_mode == 0) return 1;
        const uint32_t pk = pos_desc_key(pos[i]);
        if (pk > PK) return 1;
        if (pk < PK) return 0;
        return tie_mode == 1 ? 1 : -1;
    };
    if (tie_mode == 2) {
        row_ordered_ranks(rc, sh, lo, hi, [&](int i) { return decide(i) < 0; },
                          [&](int i, int rank) { keep[i] = (unsigned long long)rank < slot_need ? 1 : 0; });
    }
    for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
        const int d = decide(i);
        if (d >= 0) keep[i] = (uint8_t)d;
    }
    if (rc.rank == 0 && threadIdx.x == 0) a.kept[row] = nprot + room;
    rc.cl.sync();
}

}  // namespace

cudaError_t launch_select(const CacheView &c, const float *crf, const int32_t *budget, uint32_t protect,
                          uint8_t *keep, int32_t *kept, int32_t *status, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int C = row_cluster_size(c.rows, sms);
    const int per = (int)((c.max_slots + C - 1) / C);
    const int cap = per < 40960 ? per : 0;
    const size_t smem = sizeof(RowShared) + (size_t)cap * 4;
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    SelectArgs a{c, crf, budget, protect, keep, kept, status, cap};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c.rows * C));
    cfg.blockDim = dim3(kThreads);
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
