// Top-budget selection, one CTA per row.
//
// Eviction keeps the top-`budget` entries of each (sequence, layer, KV head) row by
// their LRFU value, ties broken by the lower token position, then the lower slot
// ("ActKV Dissected", Summary: LRFU eviction policy; the budget is per trajectory).
// Labels selected by protect_label_mask are always kept and use up budget first.
//
// Radix search over order-preserving fp32 keys (three digits), then over position
// keys among the entries tied at the threshold; equal (value, position) pairs are
// settled by slot order with a CTA scan.
#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 1024;

struct SelectArgs {
    CacheView c;
    const float *crf;
    const int32_t *budget;
    uint32_t protect;
    uint8_t *keep;
    int32_t *kept;
    int32_t *status;
    int cache_cap;
};

struct SelShared {
    RadixShared rs;
    int red_i[32];
};

__global__ void __launch_bounds__(kThreads) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelShared &sh = *reinterpret_cast<SelShared *>(smem_raw);
    uint32_t *kc = reinterpret_cast<uint32_t *>(smem_raw + sizeof(SelShared));

    const int row = blockIdx.x;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const int seq = row / (c.num_layers * c.num_kv_heads);
    const int B = max(a.budget[seq], 0);
    const float *crf = a.crf + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    const uint8_t *lab = c.slot_label ? c.slot_label + (int64_t)row * c.max_slots : nullptr;
    uint8_t *keep = a.keep + (int64_t)row * c.max_slots;
    const bool cached = n <= a.cache_cap;
    const uint32_t protect = lab ? a.protect : 0u;

    auto prot = [&](int i) -> bool { return protect && ((protect >> (lab[i] & 31)) & 1u); };

    int bad = 0, nprot = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float v = crf[i];
        if (!is_finite(v)) bad = 1;
        if (cached) kc[i] = float_key(v == 0.f ? 0.f : v);  // -0.0 ranks as +0.0
        nprot += prot(i) ? 1 : 0;
    }
    if (block_or(bad, sh.red_i)) {
        // keep everything on a faulted row: nothing is evicted
        for (int i = threadIdx.x; i < n; i += blockDim.x) keep[i] = 1;
        if (threadIdx.x == 0) {
            a.kept[row] = n;
            report(a.status, KVC_DEV_NONFINITE, row);
        }
        return;
    }
    nprot = block_sum<int>(nprot, sh.red_i);
    auto key = [&](int i) -> uint32_t {
        if (cached) return kc[i];
        const float v = crf[i];
        return float_key(v == 0.f ? 0.f : v);
    };
    const int ncand = n - nprot;
    const int room = min(max(B - nprot, 0), ncand);

    // mode 0: keep all candidates; 1: none; 2: threshold (+ ties)
    int mode = room >= ncand ? 0 : (room == 0 ? 1 : 2);
    uint32_t T = 0, PK = 0;
    int tie_mode = 0, slot_need = 0;
    if (mode == 2) {
        RadixResult r = radix_search_desc<false>(
            n, (unsigned long long)room, key, [](int) { return 1ull; }, [&](int i) { return !prot(i); }, sh.rs);
        T = r.key;
        const unsigned long long need = room - r.above;
        if (need < r.eq_count) {
            RadixResult r2 = radix_search_desc<false>(
                n, need, [&](int i) { return pos_desc_key(pos[i]); }, [](int) { return 1ull; },
                [&](int i) { return !prot(i) && key(i) == T; }, sh.rs);
            PK = r2.key;
            tie_mode = 1;
            const unsigned long long need2 = need - r2.above;
            if (need2 < r2.eq_count) {
                tie_mode = 2;
                slot_need = (int)need2;
            }
        }
    }
    auto decide = [&](int i) -> int {
        if (prot(i)) return 1;
        if (mode == 0) return 1;
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
    if (tie_mode != 2) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) keep[i] = (uint8_t)decide(i);
    } else {
        const int chunk = (n + blockDim.x - 1) / blockDim.x;
        const int b0 = threadIdx.x * chunk, b1 = min(n, b0 + chunk);
        int cnt = 0;
        for (int i = b0; i < b1; ++i) cnt += decide(i) < 0;
        int total;
        int rank = block_exclusive_scan(cnt, sh.red_i, &total);
        for (int i = b0; i < b1; ++i) {
            int d = decide(i);
            if (d < 0) d = (rank++ < slot_need) ? 1 : 0;
            keep[i] = (uint8_t)d;
        }
    }
    if (threadIdx.x == 0) a.kept[row] = nprot + room;
}

}  // namespace

cudaError_t launch_select(const CacheView &c, const float *crf, const int32_t *budget, uint32_t protect,
                          uint8_t *keep, int32_t *kept, int32_t *status, cudaStream_t stream) {
    const int cap = (int)(c.max_slots < 40960 ? c.max_slots : 40960);
    const size_t smem = sizeof(SelShared) + (size_t)cap * 4;
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    SelectArgs a{c, crf, budget, protect, keep, kept, status, cap};
    select_kernel<<<c.rows, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kvc
