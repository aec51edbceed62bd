// Tensor-core LSE of a query set over its row's keys (bf16 caches), sm_100a.
//
// Beacon queries ("BeaconKV ...", Key ideas) are not decoded tokens, so no attention kernel produced their
// log-sum-exp; the scoring step ("ActKV Dissected", Component 3: probabilities are logits minus the LSE) needs
// it, so this pass computes
//
//   lse[seq][layer][h][j] = ln sum_{i : slot_pos_i <= q_pos_j} exp(q_{j,h} . k_i / sqrt(D))      (-inf: no key)
//
// A cluster of S CTAs per (row, tile of 128 query columns: floor(128 / G) queries x G heads, query-major), each
// CTA a contiguous share of the row's key tiles (S is chosen on the host so the CTAs fill whole waves of SMs);
// the CTA's columns stay in shared memory (the A operand) while its keys stream through in tiles of 128 (the B
// operand, gathered page by page with TMA).  One M128 x N128 x K=D tcgen05.mma per key tile into one of four TMEM
// accumulators; 16 epilogue warps (TMEM lane quadrant = 32 columns, key quarter = 32 keys of the tile) keep a
// running (max, sum) per column in the log2 domain, merged over the quarters at the end, then over the
// cluster's CTAs through distributed shared memory.
//   warp 0  TMA: the query tile once, then per key tile its 8 pages (16 x 64 bf16 boxes, 128B swizzle).
//   warp 1  TMEM owner and MMA issuer.
//   warp 2  key decoder: per key tile the pages and the slot positions (readable keys only).
// Key tiles entirely after the last query of the CTA are skipped.  Every wait is bounded (about one second);
// on expiry the CTA records KVC_DEV_TIMEOUT, lets in-flight copies land, drains its MMAs and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>

#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

using namespace sm100;

constexpr int kCols = 128;      // query columns per CTA (MMA M)
constexpr int kKeys = 128;      // keys per tile (MMA N)
constexpr int kPages = 8;       // pages of 16 slots per key tile
constexpr int kStages = 4;      // key-tile stages
constexpr int kAcc = 4;         // TMEM accumulators (4 x 128 columns)
constexpr int kRing = 4;        // key-tile records
constexpr int kThreads = 640;
constexpr int kEpi0 = 4;
constexpr int kEpiWarps = 16;
constexpr uint64_t kTimeoutNs = 1000000000ull;

struct KeyRec {
    int32_t n_keys, kmax, last, qfull;    // last: final record of the CTA; qfull bit q: keys 32q..32q+31 readable
    int32_t page[kPages];
    int32_t kpos[kKeys];                  // INT32_MAX for a key that is absent or unreadable
};

struct Ctrl {
    uint64_t q_full, k_full[kStages], k_empty[kStages], acc_full[kAcc], acc_empty[kAcc];
    uint64_t r_full[kRing], r_empty[kRing], drain;
    uint32_t tmem_base;
    int32_t abort;
    float part_m[3][kCols], part_s[3][kCols];
    float fin_m[kCols], fin_s[kCols];     // this CTA's (max, sum) per column when a row's keys are split
};

struct LseTcArgs {
    CacheView c;
    QueryView q;
    int32_t *status;
    int nqt;           // queries per CTA tile: floor(128 / G)
    int tiles_q;       // column tiles per row
    int splits;        // CTAs (one cluster) sharing a column tile, each a contiguous run of the row's key tiles
    float scale_log2e; // log2(e) / sqrt(D)
};

template <int D>
struct LPlan {
    static constexpr int kChunks = D / 64;
    static constexpr int kQBytes = kCols * D * 2;
    static constexpr int kKBytes = kKeys * D * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffRec = kOffK + kStages * kKBytes;
    static constexpr int kOffCtrl = kOffRec + kRing * (int)sizeof(KeyRec);
    static constexpr int kBytes = kOffCtrl + (int)sizeof(Ctrl) + 1024;
    static_assert(kBytes <= 232448, "shared memory plan exceeds 227 KB per CTA");
};

__device__ bool wait_bar(uint64_t *bar, uint32_t parity, Ctrl &ctl, int32_t *status, int row) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test_sleep(bar, parity, 20000u)) return true;
        if ((it & 3) == 0) {
            if (*(volatile int32_t *)&ctl.abort) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                report(status, KVC_DEV_TIMEOUT, row);
                atomicExch(&ctl.abort, 1);
                return false;
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    lse_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q, LseTcArgs a) {
    using PL = LPlan<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + PL::kOffQ;
    uint8_t *sK = smem + PL::kOffK;
    KeyRec *rec = reinterpret_cast<KeyRec *>(smem + PL::kOffRec);
    Ctrl &ctl = *reinterpret_cast<Ctrl *>(smem + PL::kOffCtrl);

    const CacheView &c = a.c;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x % a.splits, unit = blockIdx.x / a.splits;
    const int row = unit / a.tiles_q, qt = unit % a.tiles_q;
    const int RPS = c.num_layers * c.num_kv_heads;
    const int seq = row / RPS, layer = (row / c.num_kv_heads) % c.num_layers, kvh = row % c.num_kv_heads;
    const int G = a.q.group, nqt = a.nqt;
    const int nq = min(a.q.num_q[seq], a.q.max_q);
    const int j0 = qt * nqt;
    if (j0 >= nq) return;   // no query of this tile exists (uniform across the CTA)
    const int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (qt == 0 && threadIdx.x == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        return;
    }
    if (n == 0) {
        // no keys: every column of the tile sees nothing
        for (int col = threadIdx.x; split == 0 && col < nqt * G; col += kThreads) {
            const int j = j0 + col / G;
            if (j < nq)
                a.q.lse[((int64_t)(seq * c.num_layers + layer) * a.q.num_q_heads + kvh * G + col % G) * a.q.max_q + j] =
                    -INFINITY;
        }
        return;
    }
    // latest query position of the tile: key tiles after it are skipped
    int qlast = INT32_MIN;
    for (int j = j0 + lane; j < min(nq, j0 + nqt); j += 32) qlast = max(qlast, a.q.q_pos[(int64_t)seq * a.q.max_q + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qlast = max(qlast, __shfl_xor_sync(0xffffffffu, qlast, o));

    for (int i = threadIdx.x; i < PL::kOffRec / 16; i += kThreads) reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        mbar_init(&ctl.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl.k_full[s], 1);
            mbar_init(&ctl.k_empty[s], 1);
        }
        for (int b = 0; b < kAcc; ++b) {
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], kEpiWarps);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&ctl.r_full[r], 1);
            mbar_init(&ctl.r_empty[r], 2 + kEpiWarps);   // TMA, MMA, epilogue
        }
        mbar_init(&ctl.drain, 1);
        ctl.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl.tmem_base)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const int ntiles = (n + kKeys - 1) / kKeys;
    // this CTA's key tiles: a contiguous share of the row's (a CTA with none still sends an end record)
    const int per_split = (ntiles + a.splits - 1) / a.splits;
    const int t_lo = min(ntiles, split * per_split), t_hi = min(ntiles, t_lo + per_split);

    if (warp == 2) {
        // ============================== key decoder ==============================
        uint32_t rk = 0, rph = 0;
        const int mp = c.max_pages_per_row;
        const int64_t ms = c.max_slots;
        // The raw loads of a key tile (its 8 block-table entries and 128 slot positions, indexes clamped into
        // the row) are issued one tile ahead, so their latency hides behind the previous tile's record.
        struct Raw {
            int page, kp[4];
        };
        auto load_raw = [&](int t, Raw &r) {
            r.page = c.block_table[(int64_t)row * mp + min(t * kPages + (lane & (kPages - 1)), mp - 1)];
#pragma unroll
            for (int i = 0; i < 4; ++i) r.kp[i] = c.slot_pos[(int64_t)row * ms + min((int64_t)t * kKeys + i * 32 + lane, ms - 1)];
        };
        const int t_end = max(t_hi, t_lo + 1);
        Raw cur, nxt;
        if (t_lo < t_hi) load_raw(t_lo, cur);
        for (int t = t_lo; t < t_end; ++t) {
            if (t > t_lo) cur = nxt;
            if (t + 1 < t_hi) load_raw(t + 1, nxt);
            const bool none = t >= t_hi;           // the end record of a CTA without key tiles
            const int k0 = t * kKeys, nk = none ? 0 : min(kKeys, n - k0);
            int page = -1;
            bool ok = false;
            if (!none && lane < kPages && k0 + lane * 16 < n) {
                page = cur.page;
                ok = page >= 0 && page < c.num_pages;
                if (!ok && qt == 0) report(a.status, KVC_DEV_BAD_PAGE, row);
            }
            const uint32_t okmask = __ballot_sync(0xffffffffu, ok);
            int kp[4], kmin = INT32_MAX, kmax = INT32_MIN;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int key = i * 32 + lane;
                const bool v = key < nk && ((okmask >> (key >> 4)) & 1u);
                kp[i] = v ? cur.kp[i] : INT32_MAX;
                if (v) {
                    kmin = min(kmin, kp[i]);
                    kmax = max(kmax, kp[i]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
                kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
            }
            const bool last = t == max(t_hi, t_lo + 1) - 1;
            if (kmin > qlast && !last) continue;   // no column of this CTA sees any key of the tile
            if (!wait_bar(&ctl.r_empty[rk], rph ^ 1, ctl, a.status, row)) break;
            KeyRec &R = rec[rk];
            const bool skip = kmin > qlast;        // the last tile still goes out, as the end marker
#pragma unroll
            for (int i = 0; i < 4; ++i) R.kpos[i * 32 + lane] = skip ? INT32_MAX : kp[i];
            if (lane < kPages) R.page[lane] = (ok && !skip) ? page : -1;
            if (lane == 0) {
                R.n_keys = skip ? 0 : nk;
                R.kmax = kmax;
                R.last = last ? 1 : 0;
                int qf = 0;
                for (int q = 0; q < 4; ++q)
                    if (nk >= 32 * q + 32 && ((okmask >> (2 * q)) & 3u) == 3u) qf |= 1 << q;
                R.qfull = qf;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.r_full[rk]);
            if (++rk == kRing) { rk = 0; rph ^= 1; }
        }
    } else if (warp == 0) {
        // ============================== TMA ==============================
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
        if (lane == 0) {
            mbar_expect_tx(&ctl.q_full, (uint32_t)(nqt * G) * 128u * PL::kChunks);
#pragma unroll
            for (int kc = 0; kc < PL::kChunks; ++kc)
                tma_load_4d(smem_u32(sQ + kc * (kCols * 128)), &tmap_q, &ctl.q_full, kc * 64, kvh * G, j0,
                            seq * c.num_layers + layer);
        }
        __syncwarp();
        uint32_t rk = 0, rph = 0, ks = 0, kph = 0;
        for (;;) {
            if (!wait_bar(&ctl.r_full[rk], rph, ctl, a.status, row)) break;
            const KeyRec &R = rec[rk];
            const int last = R.last;
            if (!wait_bar(&ctl.k_empty[ks], kph ^ 1, ctl, a.status, row)) break;
            const int pg = lane < kPages ? R.page[lane] : -1;
            const uint32_t m = __ballot_sync(0xffffffffu, pg >= 0);
            if (lane == 0) {
                if (m) mbar_expect_tx(&ctl.k_full[ks], (uint32_t)__popc(m) * 2048u * PL::kChunks);
                else mbar_arrive(&ctl.k_full[ks]);
            }
            __syncwarp();
            if (pg >= 0) {
#pragma unroll
                for (int kc = 0; kc < PL::kChunks; ++kc)
                    tma_load_2d(smem_u32(sK + ks * PL::kKBytes + kc * (kKeys * 128) + lane * (16 * 128)), &tmap_k,
                                &ctl.k_full[ks], kc * 64, pg * 16);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.r_empty[rk]);
            if (++rk == kRing) { rk = 0; rph ^= 1; }
            if (++ks == kStages) { ks = 0; kph ^= 1; }
            if (last) break;
        }
    } else if (warp == 1) {
        // ============================== MMA ==============================
        uint32_t rk = 0, rph = 0, ks = 0, kph = 0, ab = 0, abph = 0;
        bool issued = false;
        constexpr uint32_t kHi = desc_hi(1024, kLayoutSw128);
        constexpr uint32_t kIdesc = idesc_bf16(kCols, kKeys);
        const uint32_t q_lo = desc_lo(smem_u32(sQ)), k_lo0 = desc_lo(smem_u32(sK));
        if (wait_bar(&ctl.q_full, 0, ctl, a.status, row)) {
            for (;;) {
                if (!wait_bar(&ctl.r_full[rk], rph, ctl, a.status, row)) break;
                const int last = rec[rk].last;
                if (!wait_bar(&ctl.k_full[ks], kph, ctl, a.status, row)) break;
                if (!wait_bar(&ctl.acc_empty[ab], abph ^ 1, ctl, a.status, row)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t d = tmem + ab * kKeys;
                    const uint32_t k_lo = k_lo0 + ((ks * PL::kKBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (uint32_t)(((kk >> 2) * (kCols * 128) + (kk & 3) * 32) >> 4);
                        mma_cta(d, ((uint64_t)kHi << 32) | (q_lo + off), ((uint64_t)kHi << 32) | (k_lo + off), kIdesc,
                                kk > 0 ? 1u : 0u);
                    }
                    commit_cta(&ctl.k_empty[ks]);
                    commit_cta(&ctl.acc_full[ab]);
                }
                issued = true;
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.r_empty[rk]);
                if (++rk == kRing) { rk = 0; rph ^= 1; }
                if (++ks == kStages) { ks = 0; kph ^= 1; }
                if (++ab == kAcc) { ab = 0; abph ^= 1; }
                if (last) break;
            }
        }
        if (issued) {
            if (lane == 0) commit_cta(&ctl.drain);
            __syncwarp();
            const uint64_t t0 = now_ns();
            while (!mbar_test(&ctl.drain, 0) && now_ns() - t0 < kTimeoutNs) {}
        }
    } else if (warp >= kEpi0) {
        // ============================== epilogue ==============================
        const int quad = warp & 3, kq = (warp - kEpi0) >> 2;
        const int col = quad * 32 + lane;          // TMEM lane = query column of the tile
        const int jq = col / G, g = col % G, j = j0 + jq;
        const bool live = col < nqt * G && j < nq;
        const int qpos = live ? a.q.q_pos[(int64_t)seq * a.q.max_q + j] : INT32_MIN;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float sc = a.scale_log2e;
        float m = -INFINITY, s = 0.f;
        uint32_t rk = 0, rph = 0, ab = 0, abph = 0;
        bool ok = true;
        for (;;) {
            if (!wait_bar(&ctl.r_full[rk], rph, ctl, a.status, row)) { ok = false; break; }
            const KeyRec &R = rec[rk];
            const int last = R.last, nk = R.n_keys, kmax = R.kmax;
            if (!wait_bar(&ctl.acc_full[ab], abph, ctl, a.status, row)) { ok = false; break; }
            tc_fence_after();
            if (nk > kq * 32) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_addr + ab * kKeys + kq * 32, r);
                // every key of the quarter readable and at or before this column's position: no mask
                const bool all = ((R.qfull >> kq) & 1) && kmax <= qpos;
                const int32_t *kp = R.kpos + kq * 32;
                tmem_wait32(r);
                float lm = -INFINITY;
                if (__all_sync(0xffffffffu, all)) {
                    // no column of the warp needs the mask (decided per warp, so the masked path below costs the
                    // fast one nothing); the scaling runs as packed f32x2 products
                    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                    for (int u = 0; u < 32; u += 2) {
                        const float2 x = __fmul2_rn(make_float2(__uint_as_float(r[u]), __uint_as_float(r[u + 1])), sc2);
                        r[u] = __float_as_uint(x.x);
                        r[u + 1] = __float_as_uint(x.y);
                        lm = fmaxf(lm, fmaxf(x.x, x.y));
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        float x = __uint_as_float(r[u]) * sc;
                        const int p = kp[u];   // absent or unreadable keys hold INT32_MAX and are never visible
                        if (p > qpos || p == INT32_MAX) x = -INFINITY;
                        r[u] = __float_as_uint(x);
                        lm = fmaxf(lm, x);
                    }
                }
                if (lm != -INFINITY) {
                    const float nm = fmaxf(m, lm);
                    const float2 nm2 = make_float2(-nm, -nm);
                    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                    for (int u = 0; u < 32; u += 2) {
                        const float2 d = __fadd2_rn(make_float2(__uint_as_float(r[u]), __uint_as_float(r[u + 1])), nm2);
                        acc = __fadd2_rn(acc, make_float2(ex2(d.x), ex2(d.y)));
                    }
                    s = s * ex2(m - nm) + (acc.x + acc.y);
                    m = nm;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ctl.acc_empty[ab]);
                mbar_arrive(&ctl.r_empty[rk]);
            }
            if (++rk == kRing) { rk = 0; rph ^= 1; }
            if (++ab == kAcc) { ab = 0; abph ^= 1; }
            if (last) break;
        }
        // merge the four key quarters of each column
        if (ok && kq != 0) {
            ctl.part_m[kq - 1][col] = m;
            ctl.part_s[kq - 1][col] = s;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
        if (ok && kq == 0 && live) {
            float M = m;
            for (int u = 0; u < 3; ++u) M = fmaxf(M, ctl.part_m[u][col]);
            float S = 0.f;
            if (M != -INFINITY) {
                S = s * ex2(m - M);
                for (int u = 0; u < 3; ++u) S += ctl.part_s[u][col] * ex2(ctl.part_m[u][col] - M);
            }
            if (a.splits == 1)
                a.q.lse[((int64_t)(seq * c.num_layers + layer) * a.q.num_q_heads + kvh * G + g) * a.q.max_q + j] =
                    S > 0.f ? (M + __log2f(S)) * 0.6931471805599453f : -INFINITY;
            ctl.fin_m[col] = M;
            ctl.fin_s[col] = S;
        }
    }
    if (*(volatile int32_t *)&ctl.abort) {
        const uint64_t t0 = now_ns();
        while (now_ns() - t0 < 50000ull) {}
    }
    if (a.splits > 1) {
        // the cluster's CTAs split the row's keys: CTA 0 merges their (max, sum) per column through distributed
        // shared memory; the closing cluster barrier keeps every CTA's shared memory alive until then
        cg::cluster_group cl = cg::this_cluster();
        cl.sync();
        if (split == 0 && threadIdx.x < nqt * G) {
            const int col = threadIdx.x, j = j0 + col / G, g = col % G;
            if (j < nq) {
                float M = -INFINITY;
                for (int r = 0; r < a.splits; ++r) M = fmaxf(M, cl.map_shared_rank(&ctl, r)->fin_m[col]);
                float S = 0.f;
                if (M != -INFINITY)
                    for (int r = 0; r < a.splits; ++r) {
                        const Ctrl *p = cl.map_shared_rank(&ctl, r);
                        S += p->fin_s[col] * ex2(p->fin_m[col] - M);
                    }
                a.q.lse[((int64_t)(seq * c.num_layers + layer) * a.q.num_q_heads + kvh * G + g) * a.q.max_q + j] =
                    S > 0.f ? (M + __log2f(S)) * 0.6931471805599453f : -INFINITY;
            }
        }
        cl.sync();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

template <int D>
cudaError_t launch_lse_tc_t(const CacheView &c, const QueryView &q, int32_t *status, cudaStream_t stream) {
    using PL = LPlan<D>;
    if (!tmap_encoder()) return cudaErrorNotSupported;
    const int G = q.group, nqt = kCols / G;
    CUtensorMap tk, tq;
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)c.num_pages * 16};
        cuuint64_t strides[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, 16};
        if (tmap_bf16(kTmapLseK, &tk, 2, c.k_pool, dims, strides, box) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)q.num_q_heads, (cuuint64_t)q.max_q,
                              (cuuint64_t)c.num_seqs * c.num_layers};
        cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)q.num_q_heads * D * 2,
                                 (cuuint64_t)q.max_q * q.num_q_heads * D * 2};
        cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)nqt, 1};
        if (tmap_bf16(kTmapLseQ, &tq, 4, q.q, dims, strides, box) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    LseTcArgs args;
    args.c = c;
    args.q = q;
    args.status = status;
    args.nqt = nqt;
    args.tiles_q = (q.max_q + nqt - 1) / nqt;
    args.scale_log2e = (float)(1.4426950408889634 / std::sqrt((double)D));
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)lse_tc_kernel<D>, PL::kBytes, smem_set);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)c.rows * args.tiles_q;
    if (units <= 0) return cudaSuccess;
    // One CTA per SM: split each column tile's keys over the cluster size S (1..8) that minimises the waves of
    // CTAs per unit of work, ceil(units * S / SMs) / S, keeping at least four key tiles per CTA.
    const int sms = device_sms();
    const int64_t ntiles = (c.max_slots + kKeys - 1) / kKeys;
    int S = 1;
    double best = (double)((units + sms - 1) / sms);
    for (int t = 2; t <= 8; ++t) {
        if (ntiles < 4 * t) break;
        const double cost = (double)((units * t + sms - 1) / sms) / t;
        if (cost < best - 1e-9) {
            best = cost;
            S = t;
        }
    }
    args.splits = S;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * S));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = PL::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, lse_tc_kernel<D>, tk, tq, args);
}

}  // namespace

bool lse_tc_supported(const CacheView &c, const QueryView &q) {
    return c.dtype == KVC_BF16 && (c.head_dim == 64 || c.head_dim == 128) && c.page_size == 16 && q.group >= 1 &&
           q.group <= kCols;
}

cudaError_t launch_lse_tc(const CacheView &c, const QueryView &q, int32_t *status, cudaStream_t stream) {
    if (c.head_dim == 64) return launch_lse_tc_t<64>(c, q, status, stream);
    return launch_lse_tc_t<128>(c, q, status, stream);
}

}  // namespace kvc
