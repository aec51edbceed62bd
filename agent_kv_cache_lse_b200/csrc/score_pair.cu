// Tensor-core scoring from the LSE (bf16 caches) on pairs of SMs, sm_100a.
//
// "ActKV Dissected", Component 3: the softmax log-sum-exp is a byproduct of paged attention, so each
// query's attention probabilities are recovered as its logits minus the LSE, with no gather of the
// attention matrix and no recompute of the attention itself; Component 1: an entry's score is the
// attention tallied over the action tokens (here: over the query set and the query heads of the GQA
// group).
//
//   s[row][i] = sum_{j, g} [q_pos_j >= slot_pos_i] * 2^( log2(e)/sqrt(D) * (q_{j,g} . k_i - lse_{j,g} * sqrt(D)) )
//
// The LSE term rides in the contraction: every column's B operand gets one more K step holding
// -(lse * sqrt(D)) split into three bf16 parts (together exact to fp32 precision), met by a constant A step of
// ones, so that the accumulator already holds q.k - lse * sqrt(D) and the epilogue needs no per-column data
// wherever the causal mask is trivially all-visible.
//
// Work unit: a pair tile of 256 keys of one row, split over a cluster of two CTAs (128 keys each), times the
// visible 256-column blocks of the row's query set (query-major: column = query * G + head, the first
// half's queries in CTA 0's shared memory, the second half's in CTA 1's).  One tcgen05.mma.cta_group::2
// (M = 256, N = 256, K = 16) chain per block, issued by CTA 0, reads each CTA's keys and query half from its
// own shared memory and leaves each CTA's 128 keys x 256 columns in its own TMEM (two 256-column
// accumulator buffers).
//
// Roles per CTA (20 warps):
//   warp 0     TMA: per tile the CTA's 8 K pages (16 x 64 bf16 boxes, 128B swizzle), per visible block the
//              CTA's query half (4-D map D, head, query, seq*layer); all completing on CTA 0's barriers.
//   warp 1     TMEM owner (both CTAs) and, in CTA 0, the MMA issuer.
//   warp 2     tile decoder: row length, the pair tile's 16 block-table entries and 256 slot positions,
//              visible blocks, and per 32-key quadrant of this CTA the blocks it must mask or may skip.
//   warp 3     column warp: per visible block the LSE step of the B operand for this CTA's 128 columns and
//              the positions of all 256 columns (for blocks that straddle the causal boundary).
//   warps 4-19 epilogue: (TMEM lane quadrant, 64-column quarter); thread = key; tcgen05.ld 16 columns at a
//              time, 2^(acc * log2e/sqrt(D)) (three quarters on the MUFU unit, a quarter by polynomial on the
//              FMA pipes), causal select only in straddling blocks, register sums, quarters joined through
//              shared memory at the end of the tile.
// Every barrier wait is bounded (about one second of global time); on expiry the CTA records
// KVC_DEV_TIMEOUT, raises the abort flag in both CTAs, lets its in-flight copies land, drains its MMAs and
// leaves through the closing cluster barrier, so no CTA exits while its peer can still reach its memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace kvc {
namespace {

using namespace sm100;

constexpr int kPairKeys = 256;    // keys per pair tile
constexpr int kCtaKeys = 128;     // keys per CTA (MMA rows per CTA)
constexpr int kCtaPages = 8;      // pages of 16 slots per CTA
constexpr int kCols = 256;        // MMA N: columns per block
constexpr int kHalfCols = 128;    // columns per CTA half of a block
constexpr int kMaxBlocks = 256;   // column blocks per sequence
constexpr int kTiles = 4;         // tile ring depth
constexpr int kMaxStages = 6;     // query-half stages (D = 64; three at D = 128)
constexpr int kQp = 8;            // column-position ring depth
constexpr int kThreads = 640;     // 20 warps
constexpr int kEpi0 = 4;          // first epilogue warp
constexpr int kEpiWarps = 16;
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kBig = 1.329227995784916e36f;  // 2^120: the LSE step of an absent column (exact in bf16)

struct TileRec {
    int32_t row, seq, layer, kvh;           // row < 0: end of work
    int32_t t, n_keys, first_vis, nq;       // n_keys: this CTA's keys in the tile; first_vis < 0: nothing visible
    uint32_t okmask;                        // readable pages of the pair tile (bit p: page p, 16 pages)
    int32_t page[kCtaPages];                // this CTA's pages (-1: none)
    uint32_t vmask[kMaxBlocks / 32];        // visible blocks
    uint32_t see[4][kMaxBlocks / 32];       // per key quadrant: blocks with a query that sees one of its keys
    uint32_t fast[4][kMaxBlocks / 32];      // per key quadrant: blocks all of whose queries see all of its keys
    int32_t kpos[kCtaKeys];
    uint32_t kvalid[kCtaKeys / 32];
};

struct Ctrl {
    uint64_t a_full[2], a_empty[2];         // K tiles (a_full: CTA 0's counts both CTAs' bytes)
    uint64_t q_full[kMaxStages], q_empty[kMaxStages];  // query halves + LSE steps (q_full: CTA 0's, both CTAs)
    uint64_t acc_full[2], acc_empty[2];     // TMEM accumulators (acc_empty: CTA 0's, both epilogues)
    uint64_t qp_full[kQp], qp_empty[kQp];
    uint64_t t_full[kTiles], t_empty[kTiles];
    uint64_t part_full[2];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort;
    int32_t blk_qmin[2][kMaxBlocks], blk_qmax[2][kMaxBlocks];
    float part[2][3][kCtaKeys];
};

struct PairArgs {
    CacheView c;
    QueryView q;
    float *scores;
    int32_t *status;
    int accumulate;
    int nqh;            // queries per CTA half of a block: floor(128 / G)
    int tiles_per_row;
    int64_t total_tiles;
    float scale_log2e;  // log2(e) / sqrt(D)
    double sqrt_d;
};

// ---------------------------------------------------------------- shared memory plan
template <int D>
struct Plan {
    static constexpr int kChunks = D / 64;                   // 128-byte K chunks of a row
    static constexpr int kABytes = kCtaKeys * D * 2;         // this CTA's K tile
    static constexpr int kBBytes = kHalfCols * D * 2;        // this CTA's query half of a block
    static constexpr int kStages = D == 128 ? 3 : 6;
    static constexpr int kExtBytes = kHalfCols * 32;         // LSE step: 128 rows x 16 bf16
    static constexpr int kOffA = 0;
    static constexpr int kOffB = 2 * kABytes;
    static constexpr int kOffOnes = kOffB + kStages * kBBytes;
    static constexpr int kOffExt = kOffOnes + kCtaKeys * 32;
    static constexpr int kOffQp = kOffExt + kStages * kExtBytes;
    static constexpr int kOffTiles = kOffQp + kQp * kCols * 4;
    static constexpr int kOffCtrl = kOffTiles + kTiles * (int)sizeof(TileRec);
    static constexpr int kBytes = kOffCtrl + (int)sizeof(Ctrl) + 1024;  // + alignment slack
    static_assert(kBytes <= 232448, "shared memory plan exceeds 227 KB per CTA");
    static_assert(kOffOnes % 1024 == 0 && kOffExt % 1024 == 0, "LSE-step operands need 1024-byte alignment");
    static_assert(kStages <= kMaxStages, "stage barriers");
};

__device__ __forceinline__ int next_bit(const uint32_t *mask, int b) {
    for (int x = b + 1; x < kMaxBlocks; ++x) {
        const uint32_t w = mask[x >> 5] >> (x & 31);
        if (w == 0u) {
            x |= 31;
            continue;
        }
        return x + __ffs(w) - 1;
    }
    return -1;
}

__device__ __forceinline__ bool bit(const uint32_t *mask, int b) { return (mask[b >> 5] >> (b & 31)) & 1u; }

// Raise the abort flag in both CTAs of the pair.
__device__ __forceinline__ void raise_abort(Ctrl &ctl) {
    const uint32_t local = smem_u32(&ctl.abort);
    for (uint32_t r = 0; r < 2; ++r)
        asm volatile("st.relaxed.cluster.shared::cluster.s32 [%0], %1;" ::"r"(map_rank(local, r)), "r"(1) : "memory");
}

// Bounded wait; false when the pair is aborting or the wait gave up (then both abort flags are raised).
__device__ bool wait_bar(uint64_t *bar, uint32_t parity, Ctrl &ctl, int32_t *status, int row) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 63) == 0) {
            if (*(volatile int32_t *)&ctl.abort) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                report(status, KVC_DEV_TIMEOUT, row);
                raise_abort(ctl);
                return false;
            }
        }
    }
}

// Sixteen columns of a key's accumulator row: x = acc * log2(e)/sqrt(D) (the LSE is already in acc), causal
// select unless the block is all-visible for this warp's keys, 2^x with six of every eight exponentials on the
// MUFU unit and two on the FMA pipes, running sums in packed f32x2.  An absent column holds about -2^120 and
// adds 0 (MUFU) or 2^-126 (polynomial).
template <bool kMasked>
__device__ __forceinline__ void epi16(const uint32_t (&r)[16], const int32_t *qp, int kpos, float sc, float2 &am,
                                      float2 &ap) {
    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        float2 x01 = __fmul2_rn(make_float2(__uint_as_float(r[4 * c4 + 0]), __uint_as_float(r[4 * c4 + 1])), sc2);
        float2 x23 = __fmul2_rn(make_float2(__uint_as_float(r[4 * c4 + 2]), __uint_as_float(r[4 * c4 + 3])), sc2);
        if (kMasked) {
            const int4 p = reinterpret_cast<const int4 *>(qp)[c4];
            x01.x = p.x >= kpos ? x01.x : -INFINITY;
            x01.y = p.y >= kpos ? x01.y : -INFINITY;
            x23.x = p.z >= kpos ? x23.x : -INFINITY;
            x23.y = p.w >= kpos ? x23.y : -INFINITY;
        }
        am = __fadd2_rn(am, make_float2(ex2(x01.x), ex2(x01.y)));
        ap = __fadd2_rn(ap, (c4 & 1) ? exp2_fma2(x23) : make_float2(ex2(x23.x), ex2(x23.y)));
    }
}

// ---------------------------------------------------------------- the kernel
template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    score_pair_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                      PairArgs a) {
    using PL = Plan<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + PL::kOffA;
    uint8_t *sB = smem + PL::kOffB;
    uint8_t *sOnes = smem + PL::kOffOnes;
    uint8_t *sExt = smem + PL::kOffExt;
    int32_t *sQp = reinterpret_cast<int32_t *>(smem + PL::kOffQp);
    TileRec *trec = reinterpret_cast<TileRec *>(smem + PL::kOffTiles);
    Ctrl &ctl = *reinterpret_cast<Ctrl *>(smem + PL::kOffCtrl);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const CacheView &c = a.c;
    const int G = a.q.group, nqh = a.nqh, nqb = 2 * a.nqh;
    const int RPS = c.num_layers * c.num_kv_heads;

    // zero the operand buffers once (rows no load fills hold finite values); ones in the LSE step's A operand:
    // every row [1, 1, 1, 0, 0, 0, 0, 0] in both 16-byte halves, so that whichever half the 32-byte swizzle
    // places a column's three LSE parts in, they meet three ones
    for (int i = threadIdx.x; i < PL::kOffOnes / 16; i += kThreads) reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < kCtaKeys * 2; i += kThreads) {
        const uint32_t one = 0x3F80u;  // bf16 1.0
        reinterpret_cast<uint4 *>(sOnes)[i] = make_uint4(one | (one << 16), one, 0, 0);
    }
    for (int i = threadIdx.x; i < PL::kStages * PL::kExtBytes / 16; i += kThreads)
        reinterpret_cast<uint4 *>(sExt)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.a_full[b], 1);
            mbar_init(&ctl.a_empty[b], 1);
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], 2 * kEpiWarps);
            mbar_init(&ctl.part_full[b], 12);
        }
        for (int s = 0; s < PL::kStages; ++s) {
            mbar_init(&ctl.q_full[s], 3);   // CTA 0's TMA arrival with the byte count + both column warps
            mbar_init(&ctl.q_empty[s], 1);
        }
        for (int k = 0; k < kQp; ++k) {
            mbar_init(&ctl.qp_full[k], 1);
            mbar_init(&ctl.qp_empty[k], kEpiWarps);
        }
        for (int k = 0; k < kTiles; ++k) {
            mbar_init(&ctl.t_full[k], 1);
            mbar_init(&ctl.t_empty[k], 2 + kEpiWarps + (leader ? 1 : 0));  // TMA, column warp, epilogue, MMA
        }
        mbar_init(&ctl.drain, 1);
        ctl.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl.tmem_base)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    cluster_sync();   // barriers initialised and TMEM allocated in both CTAs before any cross-CTA traffic
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    // CTA 0's barriers as seen from this CTA (the pair's MMA and its operands synchronise there)
    const uint32_t a_full0 = map_rank(smem_u32(&ctl.a_full[0]), 0), q_full0 = map_rank(smem_u32(&ctl.q_full[0]), 0),
                   acc_empty0 = map_rank(smem_u32(&ctl.acc_empty[0]), 0);

    // pair-tile order: round k takes tiles k * npairs ... , pair p the p-th in even rounds and the
    // (npairs - 1 - p)-th in odd rounds (under a causal mask the cost falls along a row)
    auto tile_id = [&](int64_t k) -> int64_t {
        return k * npairs + ((k & 1) ? (int64_t)(npairs - 1 - pair) : (int64_t)pair);
    };

    if (warp == 2) {
        // ============================== tile decoder ==============================
        uint32_t tk = 0, tph = 0;
        int cur_seq = -1, nq = 0, nblk = 0, sbuf = 0;
        bool ok = true;
        const int mp = c.max_pages_per_row;
        const int64_t ms = c.max_slots;
        for (int64_t k = 0; ok; ++k) {
            const int64_t tid = tile_id(k);
            if (tid >= a.total_tiles) break;
            const int64_t rr = tid % RPS, rest = tid / RPS;
            const int t = (int)(rest % a.tiles_per_row), seq = (int)(rest / a.tiles_per_row);
            const int row = seq * RPS + (int)rr;
            const int n = c.row_len[row];
            if (n < 0 || n > ms) {
                if (t == 0 && lane == 0 && leader) report(a.status, KVC_DEV_BAD_LENGTH, row);
                continue;
            }
            const int k0 = t * kPairKeys;
            if (k0 >= n) continue;
            const int pair_keys = min(kPairKeys, n - k0);
            const int my0 = (int)rank * kCtaKeys;
            const int n_keys = max(0, min(kCtaKeys, pair_keys - my0));
            if (seq != cur_seq) {
                // q_pos range of every block of the sequence (blocks of nqb queries)
                cur_seq = seq;
                sbuf ^= 1;
                nq = min(a.q.num_q[seq], a.q.max_q);
                nblk = (nq + nqb - 1) / nqb;
                for (int b = lane; b < nblk; b += 32) {
                    ctl.blk_qmin[sbuf][b] = INT32_MAX;
                    ctl.blk_qmax[sbuf][b] = INT32_MIN;
                }
                __syncwarp();
                const int32_t *qrow = a.q.q_pos + (int64_t)seq * a.q.max_q;
                for (int j = lane; j < nq; j += 32) {
                    const int p = qrow[j];
                    atomicMin(&ctl.blk_qmin[sbuf][j / nqb], p);
                    atomicMax(&ctl.blk_qmax[sbuf][j / nqb], p);
                }
                __syncwarp();
            }
            // the pair tile's 16 pages (both CTAs read all of them: the byte count covers both halves)
            int page = -1;
            bool page_ok = false;
            if (lane < 16 && k0 + lane * 16 < n) {
                page = c.block_table[(int64_t)row * mp + min(t * 16 + lane, mp - 1)];
                page_ok = page >= 0 && page < c.num_pages;
                if (!page_ok && (lane >> 3) == (int)rank) report(a.status, KVC_DEV_BAD_PAGE, row);
            }
            const uint32_t okmask = __ballot_sync(0xffffffffu, page_ok) & 0xFFFFu;
            // slot positions of all 256 keys: the pair's visible blocks are decided on the whole pair tile
            int kp[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int key = i * 32 + lane;
                kp[i] = key < pair_keys ? c.slot_pos[(int64_t)row * ms + k0 + key] : INT32_MAX;
            }
            int kmin = INT32_MAX;
#pragma unroll
            for (int i = 0; i < 8; ++i) kmin = min(kmin, kp[i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            // this CTA's four quadrants (keys 32q .. 32q + 31 of its 128): range of the readable keys
            int qmin4[4], qmax4[4];
            uint32_t kval[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int key = my0 + q * 32 + lane;  // within the pair tile
                const bool v = key < pair_keys && ((okmask >> (key >> 4)) & 1u);
                kval[q] = __ballot_sync(0xffffffffu, v);
                const int mine = rank ? kp[4 + q] : kp[q];
                int mn = v ? mine : INT32_MAX, mx = v ? mine : INT32_MIN;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
                qmin4[q] = mn;
                qmax4[q] = mx;
            }
            if (!wait_bar(&ctl.t_empty[tk], tph ^ 1, ctl, a.status, row)) {
                ok = false;
                break;
            }
            TileRec &R = trec[tk];
            int first_vis = -1;
#pragma unroll
            for (int w = 0; w < kMaxBlocks / 32; ++w) {
                const int b = w * 32 + lane;
                const bool live = b < nblk;
                const int bmin = live ? ctl.blk_qmin[sbuf][b] : INT32_MAX, bmax = live ? ctl.blk_qmax[sbuf][b] : INT32_MIN;
                const uint32_t m = __ballot_sync(0xffffffffu, live && bmax >= kmin);
                if (m && first_vis < 0) first_vis = w * 32 + __ffs(m) - 1;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t s = __ballot_sync(0xffffffffu, live && bmax >= kmin && bmax >= qmin4[q] &&
                                                                      qmin4[q] != INT32_MAX);
                    const uint32_t f = __ballot_sync(0xffffffffu, live && bmax >= kmin && bmin >= qmax4[q]);
                    if (lane == 0) {
                        R.see[q][w] = s;
                        R.fast[q][w] = f;
                    }
                }
                if (lane == 0) R.vmask[w] = m;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) R.kpos[i * 32 + lane] = rank ? kp[4 + i] : kp[i];
            if (lane < 4) R.kvalid[lane] = kval[lane];
            const int my_page = __shfl_sync(0xffffffffu, page_ok ? page : -1, ((int)rank * 8 + lane) & 31);
            if (lane < kCtaPages) R.page[lane] = my_page;
            if (lane == 0) {
                R.row = row;
                R.seq = seq;
                R.layer = (int)(rr / c.num_kv_heads);
                R.kvh = (int)(rr % c.num_kv_heads);
                R.t = t;
                R.n_keys = n_keys;
                R.first_vis = first_vis;
                R.nq = nq;
                R.okmask = okmask;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.t_full[tk]);
            if (++tk == kTiles) { tk = 0; tph ^= 1; }
        }
        // end-of-work marker
        if (ok && wait_bar(&ctl.t_empty[tk], tph ^ 1, ctl, a.status, -1)) {
            if (lane == 0) {
                trec[tk].row = -1;
                mbar_arrive(&ctl.t_full[tk]);
            }
        }
    } else if (warp == 0) {
        // ============================== TMA loads ==============================
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_q)) : "memory");
        uint32_t qs = 0, qph = 0, tk = 0, tph = 0, ta = 0;
        const uint32_t q_bytes_half = (uint32_t)(nqh * G) * 128u * PL::kChunks;
        bool ok = true;
        for (;;) {
            if (!wait_bar(&ctl.t_full[tk], tph, ctl, a.status, -1)) { ok = false; break; }
            const TileRec &R = trec[tk];
            const int row = R.row;
            if (row < 0) break;
            if (R.first_vis >= 0) {
                const uint32_t abuf = ta & 1;
                if (!wait_bar(&ctl.a_empty[abuf], ((ta >> 1) & 1) ^ 1, ctl, a.status, row)) { ok = false; break; }
                ++ta;
                if (leader && lane == 0)
                    mbar_expect_tx_cluster(a_full0 + abuf * 8, (uint32_t)__popc(R.okmask) * 2048u * PL::kChunks);
                __syncwarp();
                const int my_page = lane < kCtaPages ? R.page[lane] : -1;
                if (my_page >= 0) {
#pragma unroll
                    for (int kc = 0; kc < PL::kChunks; ++kc) {
                        const uint32_t dst = smem_u32(sA + abuf * PL::kABytes + kc * (kCtaKeys * 128) + lane * (16 * 128));
                        tma_load_2d_pair(dst, &tmap_k, a_full0 + abuf * 8, kc * 64, my_page * 16);
                    }
                }
                const int zq = R.seq * c.num_layers + R.layer, h0 = R.kvh * G;
                for (int b = R.first_vis; b >= 0; b = next_bit(R.vmask, b)) {
                    if (!wait_bar(&ctl.q_empty[qs], qph ^ 1, ctl, a.status, row)) { ok = false; break; }
                    if (lane == 0) {
                        if (leader) mbar_expect_tx_cluster(q_full0 + qs * 8, 2 * q_bytes_half);
#pragma unroll
                        for (int kc = 0; kc < PL::kChunks; ++kc) {
                            const uint32_t dst = smem_u32(sB + qs * PL::kBBytes + kc * (kHalfCols * 128));
                            tma_load_4d_pair(dst, &tmap_q, q_full0 + qs * 8, kc * 64, h0, b * nqb + (int)rank * nqh, zq);
                        }
                    }
                    __syncwarp();
                    if (++qs == PL::kStages) { qs = 0; qph ^= 1; }
                }
                if (!ok) break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.t_empty[tk]);
            if (++tk == kTiles) { tk = 0; tph ^= 1; }
        }
        (void)ok;
    } else if (warp == 3) {
        // ============================== column warp ==============================
        // Per visible block: the LSE step of the B operand for this CTA's 128 columns (rows of 32 bytes,
        // 32-byte swizzle: 16-byte half h of row r sits at half h ^ ((r >> 2) & 1)), and the positions of all 256
        // columns for the epilogue's causal select.
        uint32_t qs = 0, qph = 0, tk = 0, tph = 0, pk = 0, pph = 0;
        bool ok = true;
        const int mq = a.q.max_q;
        for (;;) {
            if (!wait_bar(&ctl.t_full[tk], tph, ctl, a.status, -1)) { ok = false; break; }
            const TileRec &R = trec[tk];
            const int row = R.row;
            if (row < 0) break;
            if (R.first_vis >= 0) {
                const float *lrow = a.q.lse + ((int64_t)(R.seq * c.num_layers + R.layer) * a.q.num_q_heads + R.kvh * G) * mq;
                const int32_t *prow = a.q.q_pos + (int64_t)R.seq * mq;
                const int nq = R.nq;
                // this lane's four B rows (r = 4 * lane + i) and eight position columns (c = lane + 32 * i)
                auto load_block = [&](int b, float (&lv)[4], int (&pv)[8]) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = 4 * lane + i, jq = r / G, g = r % G;
                        const int j = b * nqb + (int)rank * nqh + jq;
                        lv[i] = (r < nqh * G && j < nq) ? lrow[(int64_t)g * mq + j] : -INFINITY;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int col = lane + 32 * i, h = col >> 7, r = col & 127, jq = r / G;
                        const int j = b * nqb + h * nqh + jq;
                        pv[i] = (r < nqh * G && j < nq) ? prow[j] : INT32_MIN;
                    }
                };
                float lv[4], lvn[4];
                int pv[8], pvn[8];
                int b = R.first_vis;
                load_block(b, lv, pv);
                while (b >= 0) {
                    const int bn = next_bit(R.vmask, b);
                    if (bn >= 0) load_block(bn, lvn, pvn);   // the next block's loads are in flight meanwhile
                    if (!wait_bar(&ctl.q_empty[qs], qph ^ 1, ctl, a.status, row)) { ok = false; break; }
                    if (!wait_bar(&ctl.qp_empty[pk], pph ^ 1, ctl, a.status, row)) { ok = false; break; }
                    uint8_t *ext = sExt + qs * PL::kExtBytes;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = 4 * lane + i;
                        float h1 = -kBig, h2 = 0.f, h3 = 0.f;
                        const float l = lv[i];
                        if (l != -INFINITY) {
                            if (!is_finite(l)) {
                                report(a.status, KVC_DEV_NONFINITE, row);
                            } else {
                                // -(lse * sqrt(D)) as three bf16 parts, each the rounding of what the previous left
                                const double v = -(double)l * a.sqrt_d;
                                const __nv_bfloat16 b1 = __double2bfloat16(v);
                                const double r1 = v - (double)__bfloat162float(b1);
                                const __nv_bfloat16 b2 = __double2bfloat16(r1);
                                const double r2 = r1 - (double)__bfloat162float(b2);
                                h1 = __bfloat162float(b1);
                                h2 = __bfloat162float(b2);
                                h3 = __bfloat162float(__double2bfloat16(r2));
                            }
                        }
                        const __nv_bfloat162 p01 = __floats2bfloat162_rn(h1, h2), p23 = __floats2bfloat162_rn(h3, 0.f);
                        const uint4 part = make_uint4(*reinterpret_cast<const uint32_t *>(&p01),
                                                      *reinterpret_cast<const uint32_t *>(&p23), 0u, 0u);
                        const int half = (r >> 2) & 1;   // the logical first half's physical place
                        reinterpret_cast<uint4 *>(ext + r * 32)[half] = part;
                        reinterpret_cast<uint4 *>(ext + r * 32)[half ^ 1] = make_uint4(0, 0, 0, 0);
                    }
                    int32_t *qp = sQp + pk * kCols;
#pragma unroll
                    for (int i = 0; i < 8; ++i) qp[lane + 32 * i] = pv[i];
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&ctl.qp_full[pk]);
                        mbar_arrive_cluster(q_full0 + qs * 8);
                    }
                    if (++qs == PL::kStages) { qs = 0; qph ^= 1; }
                    if (++pk == kQp) { pk = 0; pph ^= 1; }
                    b = bn;
#pragma unroll
                    for (int i = 0; i < 4; ++i) lv[i] = lvn[i];
#pragma unroll
                    for (int i = 0; i < 8; ++i) pv[i] = pvn[i];
                }
                if (!ok) break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.t_empty[tk]);
            if (++tk == kTiles) { tk = 0; tph ^= 1; }
        }
        (void)ok;
    } else if (warp == 1) {
        // ============================== MMA issuer (CTA 0) ==============================
        if (leader) {
            uint32_t qs = 0, qph = 0, tk = 0, tph = 0, ab = 0, abph = 0, tm = 0;
            bool issued = false;
            constexpr uint32_t kHi128 = desc_hi(1024, kLayoutSw128), kHi32 = desc_hi(256, kLayoutSw32);
            constexpr uint32_t kIdesc = idesc_bf16(2 * kCtaKeys, kCols);
            const uint32_t a_lo0 = desc_lo(smem_u32(sA)), b_lo0 = desc_lo(smem_u32(sB));
            const uint64_t ones_desc = ((uint64_t)kHi32 << 32) | desc_lo(smem_u32(sOnes));
            const uint32_t ext_lo0 = desc_lo(smem_u32(sExt));
            for (;;) {
                if (!wait_bar(&ctl.t_full[tk], tph, ctl, a.status, -1)) break;
                const TileRec &R = trec[tk];
                const int row = R.row;
                if (row < 0) break;
                bool ok = true;
                if (R.first_vis >= 0) {
                    const uint32_t abuf = tm & 1;
                    if (!wait_bar(&ctl.a_full[abuf], (tm >> 1) & 1, ctl, a.status, row)) break;
                    ++tm;
                    const uint32_t a_lo = a_lo0 + ((abuf * PL::kABytes) >> 4);
                    for (int b = R.first_vis; b >= 0;) {
                        const int bn = next_bit(R.vmask, b);
                        if (!wait_bar(&ctl.q_full[qs], qph, ctl, a.status, row)) { ok = false; break; }
                        if (!wait_bar(&ctl.acc_empty[ab], abph ^ 1, ctl, a.status, row)) { ok = false; break; }
                        tc_fence_after();
                        if (lane == 0) {
                            const uint32_t d = tmem + ab * kCols;
                            const uint32_t b_lo = b_lo0 + ((qs * PL::kBBytes) >> 4);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = (uint32_t)(((kk >> 2) * (kCtaKeys * 128) + (kk & 3) * 32) >> 4);
                                mma_pair(d, ((uint64_t)kHi128 << 32) | (a_lo + off), ((uint64_t)kHi128 << 32) | (b_lo + off),
                                         kIdesc, kk > 0 ? 1u : 0u);
                            }
                            // the LSE step last: q.k is summed first, then the large subtraction
                            const uint64_t ext_desc = ((uint64_t)kHi32 << 32) | (ext_lo0 + ((qs * PL::kExtBytes) >> 4));
                            mma_pair(d, ones_desc, ext_desc, kIdesc, 1u);
                            commit_pair(&ctl.q_empty[qs], 0x3);
                            commit_pair(&ctl.acc_full[ab], 0x3);
                            if (bn < 0) commit_pair(&ctl.a_empty[abuf], 0x3);
                        }
                        issued = true;
                        __syncwarp();
                        if (++qs == PL::kStages) { qs = 0; qph ^= 1; }
                        if (++ab == 2) { ab = 0; abph ^= 1; }
                        b = bn;
                    }
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.t_empty[tk]);
                if (++tk == kTiles) { tk = 0; tph ^= 1; }
            }
            // all MMAs issued here are complete before either CTA can leave or free TMEM
            if (issued) {
                if (lane == 0) commit_pair(&ctl.drain, 0x1);
                __syncwarp();
                const uint64_t t0 = now_ns();
                while (!mbar_test(&ctl.drain, 0) && now_ns() - t0 < kTimeoutNs) {}
            }
        }
    } else {
        // ============================== epilogue ==============================
        const int e = warp - kEpi0;
        const int quad = warp & 3, cq = e >> 2;   // TMEM lane quadrant (warp % 4), 64-column quarter
        const int key = quad * 32 + lane;          // key within this CTA's 128
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        uint32_t tk = 0, tph = 0, ab = 0, abph = 0, pk = 0, pph = 0, tcount = 0;
        const float sc = a.scale_log2e;
        bool ok = true;
        for (;;) {
            if (!wait_bar(&ctl.t_full[tk], tph, ctl, a.status, -1)) break;
            const TileRec &R = trec[tk];
            const int row = R.row;
            if (row < 0) break;
            const bool kv = (R.kvalid[quad] >> lane) & 1u;
            const int kpos = R.kpos[key];
            float *dst = a.scores + (int64_t)row * c.max_slots + (int64_t)R.t * kPairKeys + (int64_t)rank * kCtaKeys + key;
            if (R.first_vis < 0) {
                if (cq == 0 && kv && key < R.n_keys && !a.accumulate) *dst = 0.f;   // no query sees this tile
            } else {
                float2 am = make_float2(0.f, 0.f), ap = make_float2(0.f, 0.f);
                for (int b = R.first_vis; b >= 0;) {
                    const int bn = next_bit(R.vmask, b);
                    if (!wait_bar(&ctl.acc_full[ab], abph, ctl, a.status, row)) { ok = false; break; }
                    tc_fence_after();
                    if (bit(R.see[quad], b)) {
                        const uint32_t tbase = tmem + lane_addr + ab * kCols + cq * 64;
                        uint32_t ra[16], rb[16];
                        if (bit(R.fast[quad], b)) {
                            tmem_ld16(tbase, ra);
                            tmem_wait16(ra);
                            tmem_ld16(tbase + 16, rb);
                            epi16<false>(ra, nullptr, kpos, sc, am, ap);
                            tmem_wait16(rb);
                            tmem_ld16(tbase + 32, ra);
                            epi16<false>(rb, nullptr, kpos, sc, am, ap);
                            tmem_wait16(ra);
                            tmem_ld16(tbase + 48, rb);
                            epi16<false>(ra, nullptr, kpos, sc, am, ap);
                            tmem_wait16(rb);
                            epi16<false>(rb, nullptr, kpos, sc, am, ap);
                        } else {
                            // straddling block: the column positions (written before the block's operands were
                            // released to the MMA, so complete by now)
                            if (!wait_bar(&ctl.qp_full[pk], pph, ctl, a.status, row)) { ok = false; break; }
                            const int32_t *qp = sQp + pk * kCols + cq * 64;
                            tmem_ld16(tbase, ra);
                            tmem_wait16(ra);
                            tmem_ld16(tbase + 16, rb);
                            epi16<true>(ra, qp, kpos, sc, am, ap);
                            tmem_wait16(rb);
                            tmem_ld16(tbase + 32, ra);
                            epi16<true>(rb, qp + 16, kpos, sc, am, ap);
                            tmem_wait16(ra);
                            tmem_ld16(tbase + 48, rb);
                            epi16<true>(ra, qp + 32, kpos, sc, am, ap);
                            tmem_wait16(rb);
                            epi16<true>(rb, qp + 48, kpos, sc, am, ap);
                        }
                    }
                    tc_fence_before();
                    if (bn < 0) {
                        // join the four column quarters (before the accumulator is released, see below)
                        const uint32_t p = tcount & 1, ph = (tcount >> 1) & 1;
                        ++tcount;
                        if (cq != 0) {
                            ctl.part[p][cq - 1][key] = (am.x + am.y) + (ap.x + ap.y);
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&ctl.part_full[p]);
                        } else {
                            if (!wait_bar(&ctl.part_full[p], ph, ctl, a.status, row)) { ok = false; break; }
                            if (kv && key < R.n_keys) {
                                const float v = (((am.x + am.y) + (ap.x + ap.y)) + ctl.part[p][0][key]) +
                                                (ctl.part[p][1][key] + ctl.part[p][2][key]);
                                *dst = a.accumulate ? *dst + v : v;
                            }
                        }
                    }
                    // Releasing the accumulator after the quarter exchange keeps part[p] from being rewritten before
                    // it is read: its next writer must first obtain an accumulator this warp released.
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_cluster(acc_empty0 + ab * 8);
                        mbar_arrive(&ctl.qp_empty[pk]);
                    }
                    if (++ab == 2) { ab = 0; abph ^= 1; }
                    if (++pk == kQp) { pk = 0; pph ^= 1; }
                    b = bn;
                }
                if (!ok) break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.t_empty[tk]);
            if (++tk == kTiles) { tk = 0; tph ^= 1; }
        }
    }
    // leave together: nothing of either CTA is touched by its peer after this barrier
    if (*(volatile int32_t *)&ctl.abort) {
        // in-flight copies into this CTA's shared memory land well within this pause
        const uint64_t t0 = now_ns();
        while (now_ns() - t0 < 50000ull) {}
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Per device: SM count and whether the kernel's shared-memory attribute has been set (set once, not per call).
struct DeviceInfo {
    int sms = 0;
    bool attr[2] = {false, false};
};
DeviceInfo g_dev[64];

template <int D>
cudaError_t launch_pair_t(const CacheView &c, const QueryView &q, float *scores, bool accumulate, int32_t *status,
                          cudaStream_t stream, char *err, size_t errlen) {
    using PL = Plan<D>;
    auto enc = encode_tiled();
    if (!enc) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled unavailable");
        return cudaErrorNotSupported;
    }
    const int G = q.group, nqh = kHalfCols / G;
    CUtensorMap tk, tq;
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)c.num_pages * 16};
        cuuint64_t strides[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, 16};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(c.k_pool), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            snprintf(err, errlen, "K tensor map encode failed (%d)", (int)r);
            return cudaErrorInvalidValue;
        }
    }
    {
        // dimensions (D, head, query, seq*layer): a box of G heads x nqh queries lands query-major
        cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)q.num_q_heads, (cuuint64_t)q.max_q,
                              (cuuint64_t)c.num_seqs * c.num_layers};
        cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)q.num_q_heads * D * 2,
                                 (cuuint64_t)q.max_q * q.num_q_heads * D * 2};
        cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)nqh, 1};
        cuuint32_t es[4] = {1, 1, 1, 1};
        CUresult r = enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q.q), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            snprintf(err, errlen, "Q tensor map encode failed (%d)", (int)r);
            return cudaErrorInvalidValue;
        }
    }
    PairArgs args;
    args.c = c;
    args.q = q;
    args.scores = scores;
    args.status = status;
    args.accumulate = accumulate ? 1 : 0;
    args.nqh = nqh;
    args.tiles_per_row = (int)((c.max_slots + kPairKeys - 1) / kPairKeys);
    args.total_tiles = (int64_t)c.rows * args.tiles_per_row;
    args.scale_log2e = (float)(1.4426950408889634 / std::sqrt((double)D));
    args.sqrt_d = std::sqrt((double)D);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    DeviceInfo &di = g_dev[dev & 63];
    if (di.sms == 0) {
        e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    if (!di.attr[D == 128]) {
        e = cudaFuncSetAttribute(score_pair_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kBytes);
        if (e != cudaSuccess) return e;
        di.attr[D == 128] = true;
    }
    const int npairs = (int)std::max<int64_t>(1, std::min<int64_t>(di.sms / 2, args.total_tiles));
    score_pair_kernel<D><<<2 * npairs, kThreads, PL::kBytes, stream>>>(tk, tq, args);
    return cudaGetLastError();
}

}  // namespace

bool score_pair_supported(const CacheView &c, const QueryView &q) {
    if (c.dtype != KVC_BF16 || (c.head_dim != 64 && c.head_dim != 128) || c.page_size != 16) return false;
    if (q.group < 1 || q.group > kHalfCols) return false;
    const int nqb = 2 * (kHalfCols / q.group);
    return (q.max_q + nqb - 1) / nqb <= kMaxBlocks;
}

cudaError_t launch_score_pair(const CacheView &c, const QueryView &q, float *scores, bool accumulate, int32_t *status,
                              cudaStream_t stream, char *err, size_t errlen) {
    if (c.head_dim == 64) return launch_pair_t<64>(c, q, scores, accumulate, status, stream, err, errlen);
    return launch_pair_t<128>(c, q, scores, accumulate, status, stream, err, errlen);
}

}  // namespace kvc
