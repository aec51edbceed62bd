// Hit gate + LRFU update, one CTA per row.
//
// "ActKV Dissected", Component 1: the entries in the top 90% of the action
// attention are action-critical, and that hit signal replaces LRFU's hit, with
// decay coefficient lambda = 0.5.  "Top 90%" is read as cumulative attention mass:
// the hits are the shortest prefix of the order (score desc, position asc, slot asc)
// whose mass reaches hit_mass of the row's total.
//
// The threshold is found with a three-digit radix search whose per-digit masses are
// 64-bit fixed-point integers (scores scaled by a power of two so the largest is
// just under 2^48): integer atomics make the search order-independent, hence the
// result deterministic run to run.
#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 1024;

struct LrfuArgs {
    CacheView c;
    const float *scores;
    float *crf;
    float decay;      // 2^(-lambda * dt)
    float hit_mass;
    int binary;
    int32_t *status;
    int cache_cap;    // keys cached in shared memory when row_len <= cache_cap
};

struct TieShared {
    RadixShared rs;
    int red_i[32];
    unsigned long long red_u[32];
    float red_f[32];
};

__global__ void __launch_bounds__(kThreads) lrfu_kernel(LrfuArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TieShared &sh = *reinterpret_cast<TieShared *>(smem_raw);
    uint32_t *kc = reinterpret_cast<uint32_t *>(smem_raw + sizeof(TieShared));

    const int row = blockIdx.x;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    const float *s = a.scores + (int64_t)row * c.max_slots;
    float *crf = a.crf + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    const bool cached = n <= a.cache_cap;

    // pass 0: validate, cache keys, row maximum
    int bad = 0;
    float mx = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float v = s[i];
        if (!is_finite(v) || v < 0.f) bad = 1;
        mx = fmaxf(mx, v);
        if (cached) kc[i] = __float_as_uint(v);
    }
    if (block_or(bad, sh.red_i)) {
        if (threadIdx.x == 0) report(a.status, KVC_DEV_NONFINITE, row);
        return;
    }
    mx = block_max(mx, sh.red_f);
    auto sval = [&](int i) -> float { return cached ? __uint_as_float(kc[i]) : s[i]; };
    // raw fp32 bits with the sign cleared: order-preserving for the (validated) non-negative scores,
    // and -0.0 maps to the key of +0.0
    auto skey = [&](int i) -> uint32_t { return __float_as_uint(sval(i)) & 0x7fffffffu; };

    // threshold key (raw fp32 bits, order-preserving for non-negative values)
    uint32_t T = 0xffffffffu;  // no hits
    uint32_t tie_pos_key = 0;  // among key == T: keep positions whose descending key > tie_pos_key ...
    int tie_mode = 0;          // 0: all of key == T are hits, 1: by position, 2: by position then slot order
    int tie_slot_need = 0;
    if (a.hit_mass >= 1.f) {
        T = 1u;  // every positive score (bits >= 1) is a hit
        tie_mode = 0;
    } else if (mx > 0.f) {
        int E;
        frexpf(mx, &E);
        const int e = 48 - E;
        auto q = [&](int i) -> unsigned long long {
            return (unsigned long long)ldexp((double)sval(i), e);
        };
        unsigned long long part = 0;
        for (int i = threadIdx.x; i < n; i += blockDim.x) part += q(i);
        const unsigned long long Sq = block_sum<unsigned long long>(part, sh.red_u);
        unsigned long long target = (unsigned long long)ceil((double)a.hit_mass * (double)Sq);
        if (target > Sq) target = Sq;
        if (target >= 1) {
            RadixResult r = radix_search_desc<true>(
                n, target, skey, q,
                [&](int i) { return sval(i) > 0.f; }, sh.rs);
            T = r.key;
            const unsigned long long qT = (unsigned long long)ldexp((double)__uint_as_float(T), e);
            const unsigned long long rem = target - r.above;
            unsigned long long need = qT > 0 ? (rem + qT - 1) / qT : r.eq_count;
            if (need > r.eq_count) need = r.eq_count;
            if (need < r.eq_count) {
                RadixResult r2 = radix_search_desc<false>(
                    n, need, [&](int i) { return pos_desc_key(pos[i]); }, [](int) { return 1ull; },
                    [&](int i) { return skey(i) == T; }, sh.rs);
                tie_pos_key = r2.key;
                tie_mode = 1;
                const unsigned long long need2 = need - r2.above;
                if (need2 < r2.eq_count) {
                    tie_mode = 2;
                    tie_slot_need = (int)need2;
                }
            }
        }
    }

    // final pass: h = score (or 1) for hits, then crf <- h + decay * crf
    auto is_hit = [&](int i, uint32_t k) -> int {
        if (k == 0u) return 0;  // zero score is never a hit
        if (k > T) return 1;
        if (k < T) return 0;
        if (tie_mode == 0) return 1;
        const uint32_t pk = pos_desc_key(pos[i]);
        if (pk > tie_pos_key) return 1;
        if (pk < tie_pos_key) return 0;
        return tie_mode == 1 ? 1 : -1;  // -1: decided by slot order below
    };
    if (tie_mode != 2) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const float v = sval(i);
            const int hit = is_hit(i, skey(i));
            const float h = hit ? (a.binary ? 1.f : v) : 0.f;
            crf[i] = fmaf(a.decay, crf[i], h);
        }
        return;
    }
    // ordered resolution of entries equal in score and position (contiguous chunks per thread)
    const int chunk = (n + blockDim.x - 1) / blockDim.x;
    const int b0 = threadIdx.x * chunk, b1 = min(n, b0 + chunk);
    int cnt = 0;
    for (int i = b0; i < b1; ++i) cnt += is_hit(i, skey(i)) < 0;
    int total;
    int rank = block_exclusive_scan(cnt, sh.red_i, &total);
    for (int i = b0; i < b1; ++i) {
        const float v = sval(i);
        int hit = is_hit(i, skey(i));
        if (hit < 0) hit = (rank++ < tie_slot_need) ? 1 : 0;
        const float h = hit ? (a.binary ? 1.f : v) : 0.f;
        crf[i] = fmaf(a.decay, crf[i], h);
    }
}

}  // namespace

cudaError_t launch_lrfu(const CacheView &c, const float *scores, float *crf, float decay, float hit_mass,
                        bool binary, int32_t *status, cudaStream_t stream) {
    const int cap = (int)(c.max_slots < 40960 ? c.max_slots : 40960);
    const size_t smem = sizeof(TieShared) + (size_t)cap * 4;
    cudaError_t e = cudaFuncSetAttribute(lrfu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LrfuArgs a{c, scores, crf, decay, hit_mass, binary ? 1 : 0, status, cap};
    lrfu_kernel<<<c.rows, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kvc
