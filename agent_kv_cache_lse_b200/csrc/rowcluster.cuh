// Row-wide collectives for a thread-block cluster that shares one row.
//
// A row of up to a few tens of thousands of entries is split into C contiguous slices,
// one per CTA of a cluster (C = 1..8).  Cluster-wide steps (a maximum, a sum, a radix
// histogram) go through distributed shared memory: each CTA publishes its partial in a
// double-buffered slot of its own shared memory, the cluster barrier orders the writes,
// and every CTA reads all C slots and reduces them itself, so all CTAs reach identical
// decisions without a broadcast.  Each collective holds exactly one cluster barrier;
// the double buffering is safe because a slot is rewritten two collectives later, after
// the barrier of the collective in between, which no CTA passes before finishing its
// reads of the earlier one.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace kvc {

namespace cg = cooperative_groups;

constexpr int kRowBins = 256;  // 8-bit digits, 4 passes over 32-bit keys
constexpr int kRowCand = 256;  // a search whose current bin holds at most this many entries finishes on them

// Per-CTA histogram of one digit.  A mass is a fixed-point integer below 2^48, kept as three 16-bit
// chunks summed in 32-bit counters (a CTA's slice holds at most 65,536 entries, so no chunk sum can
// overflow); the cluster gather recombines them exactly in 64 bits.  Native 32-bit shared-memory atomics
// stay fast under the heavy contention of rows full of similar values, where 64-bit ones do not.
struct RowHist {
    unsigned int cnt[kRowBins];
    unsigned int wt[3][kRowBins];
};

struct RowShared {
    RowHist hist[2];
    unsigned int gcnt[kRowBins];        // cluster-wide histogram of the current pass
    unsigned long long gwt[kRowBins];
    // published scalars, double-buffered
    float xf[2];
    int xi[2][2];
    unsigned long long xu[2];
    // search state (the same in every CTA of the cluster)
    uint32_t prefix, pmask;
    unsigned long long above, remaining;
    uint32_t eq_count;
    int red_i[32];
    unsigned long long red_u[32];
    float red_f[32];
    // candidate finish: this CTA's entries of the search's current bin (published to the cluster), and every
    // CTA's gathered copy of all of them
    unsigned int ncand;
    unsigned int cn[8], cb[9];          // every rank's count, gathered, and their prefix sums
    uint32_t ck[kRowCand];
    unsigned long long cw[kRowCand];
    uint32_t gk[kRowCand];
    unsigned long long gw[kRowCand];
    uint32_t fin_key, fin_eq;
    unsigned long long fin_above;
};

struct RowCtx {
    cg::cluster_group cl;
    int rank, nranks;
    int par;  // collective counter (selects the buffer)
};

__device__ inline RowCtx row_ctx() {
    RowCtx c{cg::this_cluster(), 0, 1, 0};
    c.rank = (int)c.cl.block_rank();
    c.nranks = (int)c.cl.num_blocks();
    return c;
}

// Cluster-wide max of a float and OR of an int (one collective).
__device__ inline void row_max_or(RowCtx &rc, RowShared &sh, float &v, int &flag) {
    const float m = block_max(v, sh.red_f);
    const int f = block_or(flag, sh.red_i);
    const int b = rc.par & 1;
    if (threadIdx.x == 0) {
        sh.xf[b] = m;
        sh.xi[b][0] = f;
    }
    rc.cl.sync();
    float gm = -INFINITY;
    int gf = 0;
    for (int r = 0; r < rc.nranks; ++r) {
        RowShared *p = rc.cl.map_shared_rank(&sh, r);
        gm = fmaxf(gm, p->xf[b]);
        gf |= p->xi[b][0];
    }
    rc.par++;
    v = gm;
    flag = gf;
}

// Cluster-wide sum of an int; also returns the sum over lower ranks (exclusive prefix).
__device__ inline int row_sum_int(RowCtx &rc, RowShared &sh, int v, int *below) {
    const int s = block_sum<int>(v, sh.red_i);
    const int b = rc.par & 1;
    if (threadIdx.x == 0) sh.xi[b][1] = s;
    rc.cl.sync();
    int tot = 0, low = 0;
    for (int r = 0; r < rc.nranks; ++r) {
        const int x = rc.cl.map_shared_rank(&sh, r)->xi[b][1];
        tot += x;
        if (r < rc.rank) low += x;
    }
    rc.par++;
    if (below) *below = low;
    return tot;
}

// Cluster-wide sums of two ints (CTA totals of v0, v1), with the sums over lower ranks.
__device__ inline void row_sum_int2(RowCtx &rc, RowShared &sh, int v0, int v1, int tot[2], int below[2]) {
    const int s0 = block_sum<int>(v0, sh.red_i);
    const int s1 = block_sum<int>(v1, sh.red_i);
    const int b = rc.par & 1;
    if (threadIdx.x == 0) {
        sh.xi[b][0] = s0;
        sh.xi[b][1] = s1;
    }
    rc.cl.sync();
    tot[0] = tot[1] = below[0] = below[1] = 0;
    for (int r = 0; r < rc.nranks; ++r) {
        const RowShared *p = rc.cl.map_shared_rank(&sh, r);
        const int x0 = p->xi[b][0], x1 = p->xi[b][1];
        tot[0] += x0;
        tot[1] += x1;
        if (r < rc.rank) {
            below[0] += x0;
            below[1] += x1;
        }
    }
    rc.par++;
}

// Cluster-wide sum of an unsigned 64-bit integer.
__device__ inline unsigned long long row_sum_u64(RowCtx &rc, RowShared &sh, unsigned long long v) {
    const unsigned long long s = block_sum<unsigned long long>(v, sh.red_u);
    const int b = rc.par & 1;
    if (threadIdx.x == 0) sh.xu[b] = s;
    rc.cl.sync();
    unsigned long long tot = 0;
    for (int r = 0; r < rc.nranks; ++r) tot += rc.cl.map_shared_rank(&sh, r)->xu[b];
    rc.par++;
    return tot;
}

// End of a mass-weighted radix search once the current bin (keys matching sh.prefix under sh.pmask) holds at
// most kRowCand valid entries cluster-wide: every CTA lists its entries of the bin, the cluster barrier publishes the lists,
// and every CTA gathers all of them (rank order) and finds the threshold itself: the key T whose weight
// interval (above(T), above(T) + weight(== T)] in descending key order holds the remaining target.  Each
// entry's interval is found by one pass over the gathered list (at most kRowCand x kRowCand steps), so the
// result is exact and the same in every CTA.  Saves the remaining radix passes (each a sweep, a barrier and
// a gather of four histograms).
template <bool kMass, typename KeyFn, typename WeightFn, typename ValidFn>
__device__ void row_finish_candidates(RowCtx &rc, RowShared &sh, int lo, int hi, KeyFn key, WeightFn weight,
                                      ValidFn valid) {
    const int tid = threadIdx.x;
    const uint32_t prefix = sh.prefix, pmask = sh.pmask;
    if (tid == 0) sh.ncand = 0;
    __syncthreads();
    for (int i = lo + tid; i < hi; i += blockDim.x) {
        if (!valid(i)) continue;
        const uint32_t k = key(i);
        if ((k & pmask) != prefix) continue;
        const unsigned at = atomicAdd(&sh.ncand, 1u);   // below kRowCand: the bin's count bounds it
        sh.ck[at] = k;
        sh.cw[at] = kMass ? (unsigned long long)weight(i) : 1ull;
    }
    rc.cl.sync();
    // the ranks' counts first (one remote load each, side by side), then every entry of every rank, each thread
    // loading its share with all its loads in flight
    if (tid < rc.nranks) sh.cn[tid] = rc.cl.map_shared_rank(&sh, tid)->ncand;
    __syncthreads();
    if (tid == 0) {
        unsigned int b = 0;
        for (int r = 0; r < rc.nranks; ++r) {
            sh.cb[r] = b;
            b += sh.cn[r];
        }
        sh.cb[rc.nranks] = b;
    }
    __syncthreads();
    const int nc = (int)sh.cb[rc.nranks];
    for (int e = tid; e < rc.nranks * kRowCand; e += blockDim.x) {
        const int r = e / kRowCand, j = e % kRowCand;
        if (j < (int)sh.cn[r]) {
            const RowShared *p = rc.cl.map_shared_rank(&sh, r);
            sh.gk[sh.cb[r] + j] = p->ck[j];
            sh.gw[sh.cb[r] + j] = p->cw[j];
        }
    }
    __syncthreads();
    const unsigned long long rem = sh.remaining;
    for (int i = tid; i < nc; i += blockDim.x) {
        const uint32_t ki = sh.gk[i];
        unsigned long long above = 0, eqw = 0;
        uint32_t eqc = 0;
        for (int j = 0; j < nc; ++j) {
            const uint32_t kj = sh.gk[j];
            const unsigned long long w = sh.gw[j];
            if (kj > ki) {
                above += w;
            } else if (kj == ki) {
                eqw += w;
                ++eqc;
            }
        }
        if (above < rem && rem <= above + eqw) {   // one key qualifies; its copies write the same values
            sh.fin_key = ki;
            sh.fin_above = above;
            sh.fin_eq = eqc;
        }
    }
    __syncthreads();
    if (tid == 0) {
        sh.prefix = sh.fin_key;
        sh.above += sh.fin_above;
        sh.eq_count = sh.fin_eq;
    }
    __syncthreads();
}

// Radix search over the cluster's row, from the most significant 8-bit digit down.  Finds the key T
// at which the running weight of the valid keys in descending key order first reaches `target`
// (>= 1, <= total weight); weight is 1 (count mode) or a fixed-point mass (mass mode).  The slice of
// this CTA is [lo, hi).  Same result in every thread of every CTA:
//   key = T, above = total weight of valid keys > T, eq_count = number of valid keys == T.
template <bool kMass, typename KeyFn, typename WeightFn, typename ValidFn>
__device__ RadixResult row_radix_desc(RowCtx &rc, RowShared &sh, int lo, int hi, unsigned long long target,
                                      KeyFn key, WeightFn weight, ValidFn valid) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) {
        sh.prefix = 0;
        sh.pmask = 0;
        sh.above = 0;
        sh.remaining = target;
        sh.eq_count = 0;
    }
    auto zero_hist = [&](RowHist &z) {
        for (int i = tid; i < kRowBins; i += blockDim.x) {
            z.cnt[i] = 0;
            if (kMass) z.wt[0][i] = z.wt[1][i] = z.wt[2][i] = 0;
        }
    };
    zero_hist(sh.hist[rc.par & 1]);
    __syncthreads();
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        const int b = rc.par & 1;
        RowHist &h = sh.hist[b];
        const uint32_t prefix = sh.prefix, pmask = sh.pmask;
        const int span = hi - lo;
        const int nround = (span + blockDim.x - 1) / blockDim.x * blockDim.x;
        for (int off = tid; off < nround; off += blockDim.x) {
            const int i = lo + off;
            bool in = false;
            uint32_t k = 0;
            unsigned long long wv = 0;
            if (off < span && valid(i)) {
                k = key(i);
                in = (k & pmask) == prefix;
                if (kMass && in) wv = weight(i);
            }
            const unsigned active = __ballot_sync(0xffffffffu, in);
            if (active == 0u) continue;
            // a warp whose taking part lanes all share one digit (the common case: rows full of equal or
            // similar values) adds with one atomic; otherwise every lane adds its own
            const uint32_t bin = (k >> shift) & (kRowBins - 1);
            const int first = __ffs(active) - 1;
            const uint32_t bin0 = __shfl_sync(0xffffffffu, bin, first);
            const bool uniform = __all_sync(0xffffffffu, !in || bin == bin0);
            if (uniform) {
                if (kMass) {
                    // chunk sums of the warp (each below 2^21), added once
                    unsigned int c0 = (unsigned)(wv & 0xffffu), c1 = (unsigned)((wv >> 16) & 0xffffu),
                                 c2 = (unsigned)(wv >> 32);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        c0 += __shfl_xor_sync(0xffffffffu, c0, o);
                        c1 += __shfl_xor_sync(0xffffffffu, c1, o);
                        c2 += __shfl_xor_sync(0xffffffffu, c2, o);
                    }
                    if (lane == first) {
                        atomicAdd(&h.wt[0][bin0], c0);
                        atomicAdd(&h.wt[1][bin0], c1);
                        atomicAdd(&h.wt[2][bin0], c2);
                    }
                }
                if (lane == first) atomicAdd(&h.cnt[bin0], (unsigned)__popc(active));
            } else if (in) {
                atomicAdd(&h.cnt[bin], 1u);
                if (kMass) {
                    atomicAdd(&h.wt[0][bin], (unsigned)(wv & 0xffffu));
                    atomicAdd(&h.wt[1][bin], (unsigned)((wv >> 16) & 0xffffu));
                    atomicAdd(&h.wt[2][bin], (unsigned)(wv >> 32));
                }
            }
        }
        rc.cl.sync();
        // the other buffer was last read by the peers before this barrier: clear it for the next pass now
        if (pass < 3) zero_hist(sh.hist[b ^ 1]);
        for (int i = tid; i < kRowBins; i += blockDim.x) {
            unsigned int c = 0;
            unsigned long long w = 0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {  // all remote reads issued before the sums need them
                if (r < rc.nranks) {
                    const RowHist &rh = rc.cl.map_shared_rank(&sh, r)->hist[b];
                    c += rh.cnt[i];
                    if (kMass)
                        w += (unsigned long long)rh.wt[0][i] + ((unsigned long long)rh.wt[1][i] << 16) +
                             ((unsigned long long)rh.wt[2][i] << 32);
                }
            }
            sh.gcnt[i] = c;
            sh.gwt[i] = kMass ? w : (unsigned long long)c;
        }
        rc.par++;
        __syncthreads();
        if (tid < 32) {
            constexpr int per = kRowBins / 32;
            const int top = kRowBins - 1 - lane * per;  // bins top, top-1, ..., top-per+1
            unsigned long long mine = 0;
#pragma unroll
            for (int q = 0; q < per; ++q) mine += sh.gwt[top - q];
            unsigned long long incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned long long excl = incl - mine, rem = sh.remaining;
            const bool here = excl < rem && incl >= rem;
            const unsigned who = __ballot_sync(0xffffffffu, here);
            if (here && lane == __ffs(who) - 1) {
                unsigned long long run = excl;
                for (int q = 0; q < per; ++q) {
                    const int bin = top - q;
                    const unsigned long long w = sh.gwt[bin];
                    if (run + w >= rem) {
                        sh.above += run;
                        sh.remaining = rem - run;
                        sh.prefix |= (uint32_t)bin << shift;
                        sh.pmask |= (uint32_t)(kRowBins - 1) << shift;
                        sh.eq_count = sh.gcnt[bin];
                        break;
                    }
                    run += w;
                }
            }
        }
        __syncthreads();
        if (kMass && pass < 3 && sh.eq_count <= (uint32_t)kRowCand) {   // (count passes are cheaper than the finish)
            row_finish_candidates<kMass>(rc, sh, lo, hi, key, weight, valid);
            break;
        }
    }
    RadixResult r;
    r.key = sh.prefix;
    r.above = sh.above;
    r.eq_count = sh.eq_count;
    __syncthreads();
    return r;
}

// Rank, in slot order over the whole row, of the entries flagged by amb(i) (contiguous chunks per
// thread, slices in rank order); calls out(i, rank) for each flagged entry.
template <typename AmbFn, typename OutFn>
__device__ void row_ordered_ranks(RowCtx &rc, RowShared &sh, int lo, int hi, AmbFn amb, OutFn out) {
    const int span = hi - lo;
    const int chunk = (span + blockDim.x - 1) / blockDim.x;
    const int b0 = lo + min(span, (int)threadIdx.x * chunk), b1 = lo + min(span, ((int)threadIdx.x + 1) * chunk);
    int cnt = 0;
    for (int i = b0; i < b1; ++i) cnt += amb(i) ? 1 : 0;
    int total;
    int rank = block_exclusive_scan(cnt, sh.red_i, &total);
    int below = 0;
    row_sum_int(rc, sh, cnt, &below);
    rank += below;
    for (int i = b0; i < b1; ++i)
        if (amb(i)) out(i, rank++);
}

// CTAs per row: the largest power of two up to 8 that keeps the launch (rows x c CTAs) within one wave.  A row
// kernel's 512 threads hold over half of an SM's registers, so one CTA runs per SM; a second wave would wait
// for the first one's slowest row.
__host__ inline int row_cluster_size(int rows, int sms) {
    int c = 1;
    while (c < 8 && (int64_t)rows * c * 2 <= (int64_t)sms) c <<= 1;
    return c;
}

}  // namespace kvc
