// Per-row bodies of the LRFU update, the top-budget selection and the slot plan, shared by their own kernels
// and by the fused kernels that run two of them in one launch.  Each body is one CTA's part of a cluster that
// shares a row (rowcluster.cuh); a fused kernel calls them back to back with the same cluster context.
#pragma once

#include "internal.h"
#include "rowcluster.cuh"

namespace kvc {

constexpr int kRowThreads = 512;

struct LrfuArgs {
    CacheView c;
    const float *scores;
    float *crf;
    float decay;      // 2^(-lambda * dt)
    float hit_mass;
    int binary;
    int32_t *status;
    int slice_cap;    // scores cached in shared memory when a CTA's slice fits
    int weight_cap;   // fixed-point masses cached too when the slice fits this
};

struct PlanArgs {
    CacheView c;
    const uint8_t *keep;
    const int32_t *kept;
    int32_t *move_src;
    int32_t *move_dst;
    int32_t *num_moves;
    int32_t *status;
};

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

// Hit gate + LRFU update of this CTA's slice of its row.
__device__ inline void lrfu_row(const LrfuArgs &a, RowCtx &rc, unsigned char *smem_raw) {
    RowShared &sh = *reinterpret_cast<RowShared *>(smem_raw);
    uint32_t *kc = reinterpret_cast<uint32_t *>(smem_raw + sizeof(RowShared));
    unsigned long long *qw = reinterpret_cast<unsigned long long *>(
        smem_raw + sizeof(RowShared) + (((size_t)a.slice_cap * 4 + 15) & ~(size_t)15));
    const int row = blockIdx.x / rc.nranks;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (rc.rank == 0 && threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;  // uniform across the cluster: no collective has started
    }
    const int per = (n + rc.nranks - 1) / rc.nranks;
    const int lo = min(n, rc.rank * per), hi = min(n, lo + per);
    const float *s = a.scores + (int64_t)row * c.max_slots;
    float *crf = a.crf + (int64_t)row * c.max_slots;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots;
    const bool cached = per <= a.slice_cap;
    const bool wcached = cached && per <= a.weight_cap;

    // stage the slice (raw fp32 bits, sign cleared so -0.0 ranks as 0), validate, row maximum
    int bad = 0;
    float mx = 0.f;
    for (int base = lo + threadIdx.x; base < hi; base += 8 * blockDim.x) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // eight independent loads in flight before any is used
            const int i = base + u * blockDim.x;
            v[u] = i < hi ? s[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * blockDim.x;
            if (i < hi) {
                if (!is_finite(v[u]) || v[u] < 0.f) bad = 1;
                mx = fmaxf(mx, v[u]);
                if (cached) kc[i - lo] = __float_as_uint(v[u]) & 0x7fffffffu;
            }
        }
    }
    row_max_or(rc, sh, mx, bad);
    if (bad) {
        if (rc.rank == 0 && threadIdx.x == 0) report(a.status, KVC_DEV_NONFINITE, row);
        rc.cl.sync();
        return;
    }
    auto skey = [&](int i) -> uint32_t { return cached ? kc[i - lo] : (__float_as_uint(s[i]) & 0x7fffffffu); };
    auto sval = [&](int i) -> float { return __uint_as_float(skey(i)); };

    uint32_t T = 0xffffffffu;  // threshold key; 0xffffffff: no hits
    uint32_t PK = 0;
    int tie_mode = 0;          // 0: every key == T is a hit; 1: decided by position; 2: then by slot order
    unsigned long long slot_need = 0;
    if (a.hit_mass >= 1.f) {
        T = 1u;                // every positive score is a hit
    } else if (mx > 0.f) {
        int E;
        frexpf(mx, &E);
        const int e = 48 - E;
        auto q = [&](int i) -> unsigned long long { return (unsigned long long)ldexp((double)sval(i), e); };
        unsigned long long part = 0;
        for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
            const unsigned long long w = q(i);
            part += w;
            if (wcached) qw[i - lo] = w;  // each pass of the search below reads it instead of recomputing
        }
        const unsigned long long Sq = row_sum_u64(rc, sh, part);  // its cluster barrier also orders qw
        auto qv = [&](int i) -> unsigned long long { return wcached ? qw[i - lo] : q(i); };
        unsigned long long target = (unsigned long long)ceil((double)a.hit_mass * (double)Sq);
        if (target > Sq) target = Sq;
        if (target >= 1) {
            const RadixResult r = row_radix_desc<true>(rc, sh, lo, hi, target, skey, qv,
                                                       [&](int i) { return skey(i) != 0u; });
            T = r.key;
            const unsigned long long qT = (unsigned long long)ldexp((double)__uint_as_float(T), e);
            const unsigned long long rem = target - r.above;
            unsigned long long need = qT > 0 ? (rem + qT - 1) / qT : r.eq_count;
            if (need > r.eq_count) need = r.eq_count;
            if (need < r.eq_count) {
                const RadixResult r2 = row_radix_desc<false>(
                    rc, sh, lo, hi, need, [&](int i) { return pos_desc_key(pos[i]); }, [](int) { return 1ull; },
                    [&](int i) { return skey(i) == T; });
                PK = r2.key;
                tie_mode = 1;
                const unsigned long long need2 = need - r2.above;
                if (need2 < r2.eq_count) {
                    tie_mode = 2;
                    slot_need = need2;
                }
            }
        }
    }
    auto is_hit = [&](int i) -> int {
        const uint32_t k = skey(i);
        if (k == 0u) return 0;
        if (k > T) return 1;
        if (k < T) return 0;
        if (tie_mode == 0) return 1;
        const uint32_t pk = pos_desc_key(pos[i]);
        if (pk > PK) return 1;
        if (pk < PK) return 0;
        return tie_mode == 1 ? 1 : -1;
    };
    auto update = [&](int i, int hit) {
        const float h = hit ? (a.binary ? 1.f : sval(i)) : 0.f;
        crf[i] = fmaf(a.decay, crf[i], h);
    };
    if (tie_mode == 2) {
        // entries equal in score and position: the first ones in slot order, across the cluster
        row_ordered_ranks(rc, sh, lo, hi, [&](int i) { return is_hit(i) < 0; },
                          [&](int i, int rank) { update(i, (unsigned long long)rank < slot_need); });
    }
    for (int base = lo + threadIdx.x; base < hi; base += 8 * blockDim.x) {
        float old[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * blockDim.x;
            old[u] = i < hi ? crf[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * blockDim.x;
            if (i < hi) {
                const int hit = is_hit(i);
                if (hit >= 0) crf[i] = fmaf(a.decay, old[u], hit ? (a.binary ? 1.f : sval(i)) : 0.f);
            }
        }
    }
    rc.cl.sync();  // peers may still read this CTA's shared memory
}

// Top-budget selection of this CTA's slice of its row.
__device__ inline void select_row(const SelectArgs &a, RowCtx &rc, unsigned char *smem_raw) {
    RowShared &sh = *reinterpret_cast<RowShared *>(smem_raw);
    uint32_t *kc = reinterpret_cast<uint32_t *>(smem_raw + sizeof(RowShared));
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



// Conflict-free slot plan of this CTA's slice of its row ("ActKV Dissected", Component 3): survivor j at or
// after m = kept (ascending) fills hole j before m (ascending).  Every thread owns a contiguous run of slots; a
// CTA scan plus the cluster-wide sums of the lower slices give every hole and survivor its rank, its index in
// the move list.  A rejected row gets num_moves = -1, which the compaction reads as "leave this row as it is".
__device__ inline void plan_row(const PlanArgs &a, RowCtx &rc, RowShared &sh) {
    const int row = blockIdx.x / rc.nranks;
    const CacheView &c = a.c;
    const int n = c.row_len[row];
    const int m = a.kept[row];
    if (n < 0 || n > c.max_slots || m < 0 || m > n) {
        if (rc.rank == 0 && threadIdx.x == 0) {
            a.num_moves[row] = -1;
            report(a.status, (n < 0 || n > c.max_slots) ? KVC_DEV_BAD_LENGTH : KVC_DEV_KEPT_MISMATCH, row);
        }
        return;  // uniform across the cluster: no collective has started
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

}  // namespace kvc
