// Tensor-core scoring from the LSE (bf16 caches), sm_100a.
//
// "ActKV Dissected", Component 3: the softmax log-sum-exp is a byproduct of paged
// attention, so each query's attention probabilities are recovered as its logits
// minus the LSE, with no gather of the attention matrix and no recompute of the
// attention itself; Component 1: an entry's score is the attention tallied over all
// action tokens (here: over the query set and the query heads of the GQA group).
//
//   s[row][i] = sum_{j, g} [q_pos_j >= slot_pos_i] * 2^( (q_{j,g} . k_i) * log2(e)/sqrt(D)
//                                                      - lse_{j,g} * log2(e) )
//
// Design (one persistent CTA per SM, 19 warps):
//   warp 2     decoder: per 256-key tile (one tile ahead), the row length, block-table
//              entries and slot positions, the keys' position range and with it the
//              visible column blocks; a tile record goes to the TMA warp through a ring.
//              Per visible 128-column block (query, head) of the query set, the raw column
//              data (lse, q_pos) is copied a block ahead with cp.async into a staging slot,
//              converted (four columns per lane, 16-byte shared-memory accesses, no
//              shuffles) and published through a metadata ring with the block's q_pos range
//              and, once per tile, the keys' positions.
//   warp 0     TMA: per tile record, 16 page loads (one 16x64 bf16 box per page and
//              64-column half of D) gather the K tile from the paged pool into a
//              128B-swizzled A operand; per visible block, the Q block (4-D map: D, query,
//              head, seq*layer, so that a block lands head-major: column n = g * nqb + query)
//              into a stage ring.
//   warp 1     TMEM owner and MMA issuer: for each block, two M=128 x N=128 x K=D
//              tcgen05.mma (kind::f16, bf16 in, fp32 accumulate) into one of two TMEM
//              accumulator buffers (4 x 128 of the 512 columns).
//   warps 3-18 epilogue: (TMEM lane quadrant, key half, column half); thread = key;
//              tcgen05.ld 16 columns at a time (double-buffered), x = acc * log2e/sqrt(D)
//              - lse_col * log2e in packed f32x2 arithmetic, causal select, 2^x (three
//              quarters on the MUFU unit, a quarter by polynomial on the FMA pipes), sums in
//              registers.  The two column halves of a key are added through shared memory
//              at the end of the tile; one coalesced store per key per tile.
// Blocks whose queries all precede the tile's first key are skipped entirely
// (no load, no MMA, no epilogue work).  Every barrier wait is bounded (about one
// second of global time); on expiry the kernel records KVC_DEV_TIMEOUT, drains its
// own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>

#include "common.cuh"
#include "internal.h"
#include "tmap.h"

namespace kvc {
namespace {

constexpr int kTileKeys = 256;          // keys per tile (two M=128 MMAs)
constexpr int kPagesPerTile = 16;       // page_size 16
constexpr int kCols = 128;              // MMA N: query columns per block
constexpr int kMeta = 8;                // metadata ring depth
constexpr int kMaxBlocks = 256;         // column blocks per sequence
constexpr int kTiles = 4;               // tile ring depth (decoder -> TMA warp)
constexpr int kThreads = 608;           // 19 warps: TMA, MMA, decoder, 16 epilogue
constexpr int kEpiWarps = 16;
constexpr uint64_t kTimeoutNs = 1000000000ull;

struct alignas(16) Item {
    float nL[kCols];                    // -lse * log2(e) per column (-inf for an absent column)
    int32_t qp[kCols];                  // q_pos per column (INT32_MIN for an absent column)
    int32_t kpos[kTileKeys];            // FIRST items: slot_pos of the tile's keys
    uint32_t kvalid[8];                 // FIRST items: keys that are present and readable
    int32_t row, tile, blk, flags;      // blk < 0: tile with no visible block; row < 0: end of work
    int32_t n_keys, chunks, qmin, qmax; // chunks: bit c set when 32-column chunk c has a present column;
                                        // qmin/qmax: q_pos range of the block's queries
};
static_assert(sizeof(Item) % 16 == 0, "items hold float4-read arrays");
constexpr int kFirst = 1, kLast = 2;

// A tile as the TMA warp needs it: where its pages are and which column blocks it loads Q for.
struct TileRec {
    int32_t row, seq, layer, kvh;                 // row < 0: end of work
    uint32_t okmask;                              // pages that are present and readable
    int32_t first_vis, pad0, pad1;
    int32_t page[kPagesPerTile];                  // physical page of each of the tile's 16 pages (-1: none)
    uint32_t vmask[kMaxBlocks / 32];              // visible column blocks
};

// A tile as the decoder works through it (the current one in registers, the next one in shared memory).
struct Tile {
    int row, t, n_keys, first_vis, last_vis, nq, sbuf, pad;
    const float *lrow;    // lse of the group's first head (sequence, layer, KV head)
    const int32_t *prow;  // q_pos of the sequence
};

// Raw column data of one block as copied from global memory: lse in column order, q_pos by query.
struct alignas(16) ColStage {
    float lse[kCols];
    int32_t qpos[kCols];
};

struct Ctrl {
    uint64_t q_full[8], q_empty[8];
    uint64_t a_full[2], a_empty[2];        // double-buffered K tile
    uint64_t acc_full[2], acc_empty[2];
    uint64_t m_full[kMeta], m_empty[kMeta];
    uint64_t part_full[2];                 // column-half partial sums of a tile, double-buffered
    uint64_t t_full[kTiles], t_empty[kTiles];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort;
    int32_t blk_qmin[2][kMaxBlocks], blk_qmax[2][kMaxBlocks];  // q_pos range per block, two sequences
    float part[2][kTileKeys];
    int32_t kstage[2][kTileKeys];     // producer: key positions of the current and the next tile
    uint32_t kvstage[2][8];           // producer: their readable-key masks
    uint32_t vstage[2][kMaxBlocks / 32];  // producer: their visible-block masks
    TileRec trec[kTiles];             // tile ring
    Tile tnext;                       // decoder: the tile decoded ahead
    ColStage colstage[4];             // producer: staged raw column data of upcoming blocks
};

struct TcArgs {
    CacheView c;
    QueryView q;
    float *scores;
    int32_t *status;
    int accumulate;
    int vec;           // lse / q_pos rows are 16-byte aligned and nqb % 4 == 0: 16-byte column copies
    int nqb;           // queries per column block (floor(128 / G))
    int tiles_per_row;
    int64_t total_tiles;
    float scale_log2e; // log2(e) / sqrt(D)
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait; false when the CTA is aborting or the wait gave up (then the abort flag is set).
__device__ bool mbar_wait(uint64_t *bar, uint32_t parity, Ctrl &ctl, int32_t *status, int row) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 63) == 0) {
            if (*(volatile int32_t *)&ctl.abort) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                report(status, KVC_DEV_TIMEOUT, row);
                atomicExch(&ctl.abort, 1);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// Shared-memory matrix descriptor of a 128B-swizzled K-major operand (8-row groups 1024 bytes apart, version 1,
// layout SWIZZLE_128B), split in two words: the high word is the same for every operand here, the low word
// holds the start address (in 16-byte units, 14 bits) and the leading byte offset (1).  Offsets within one
// operand buffer are added to the low word directly: addresses stay below 2^18, so the field never carries.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t addr) { return ((addr >> 4) & 0x3FFF) | (1u << 16); }

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kCols >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

template <bool kAccumulate>
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo) {
    const uint64_t ad = ((uint64_t)kDescHi << 32) | a_lo, bd = ((uint64_t)kDescHi << 32) | b_lo;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(ad), "l"(bd), "r"(kIdesc), "n"(kAccumulate ? 1 : 0));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
        "[%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Waits for this thread's TMEM loads; naming the registers of the load being waited for keeps the compiler from
// reading them before the wait.
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipes for a pair of arguments: x = n + f, n = round(x), f in [-1/2, 1/2]; 2^f by a
// degree-5 polynomial whose coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez
// exchange, derived by exp2_poly.py beside this file: 2.4e-7 relative in fp32 Horner form, the accuracy
// class of the MUFU unit's approximation, so that the two kinds of exponential are interchangeable under a
// 1e-4 ranking tolerance); 2^n enters through the exponent bits.  x is clamped at -126 so the exponent
// arithmetic stays in range (the result is then ~1e-38).  The floating-point steps run as packed f32x2
// operations.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    constexpr float kC0 = 1.0000001192092896f, kC1 = 0.6931469440460205f, kC2 = 0.24022120237350464f,
                    kC3 = 0.05550713092088699f, kC4 = 0.009675540961325169f, kC5 = 0.0013276472454890609f;
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
    x.x = fmaxf(x.x, -126.0f);
    x.y = fmaxf(x.y, -126.0f);
    const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
    const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));
    const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
    float2 p = __ffma2_rn(make_float2(kC5, kC5), f, make_float2(kC4, kC4));
    p = __ffma2_rn(p, f, make_float2(kC3, kC3));
    p = __ffma2_rn(p, f, make_float2(kC2, kC2));
    p = __ffma2_rn(p, f, make_float2(kC1, kC1));
    p = __ffma2_rn(p, f, make_float2(kC0, kC0));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Sixteen columns of a key's accumulator row: x = acc * log2(e)/sqrt(D) - lse_col * log2(e), causal select
// (unless every column of the block sees every key of the warp), 2^x, running sums.  Columns go in pairs
// through packed f32x2 arithmetic; of every eight exponentials, six run on the MUFU unit and two on the FMA
// pipes (the MUFU unit is the scarcer resource, issue slots the next one).  An absent column has
// -lse = -inf: it adds 0 (MUFU) or 2^-126 (polynomial), both far below any tolerance.
__device__ __forceinline__ void epi16(const uint32_t (&r)[16], const float *nL, const int32_t *qp, int kpos, float sc,
                                      bool fast, float2 &am, float2 &ap) {
    const float4 *L4 = reinterpret_cast<const float4 *>(nL);
    const float2 sc2 = make_float2(sc, sc);
    if (fast) {
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const float4 l = L4[c4];
            const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(r[4 * c4 + 0]), __uint_as_float(r[4 * c4 + 1])),
                                          sc2, make_float2(l.x, l.y));
            const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(r[4 * c4 + 2]), __uint_as_float(r[4 * c4 + 3])),
                                          sc2, make_float2(l.z, l.w));
            am = __fadd2_rn(am, make_float2(ex2(x01.x), ex2(x01.y)));
            ap = __fadd2_rn(ap, (c4 & 1) ? exp2_fma2(x23) : make_float2(ex2(x23.x), ex2(x23.y)));
        }
    } else {
        const int4 *P4 = reinterpret_cast<const int4 *>(qp);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const float4 l = L4[c4];
            const int4 p = P4[c4];
            float2 x01 = __ffma2_rn(make_float2(__uint_as_float(r[4 * c4 + 0]), __uint_as_float(r[4 * c4 + 1])), sc2,
                                    make_float2(l.x, l.y));
            float2 x23 = __ffma2_rn(make_float2(__uint_as_float(r[4 * c4 + 2]), __uint_as_float(r[4 * c4 + 3])), sc2,
                                    make_float2(l.z, l.w));
            x01.x = p.x >= kpos ? x01.x : -INFINITY;
            x01.y = p.y >= kpos ? x01.y : -INFINITY;
            x23.x = p.z >= kpos ? x23.x : -INFINITY;
            x23.y = p.w >= kpos ? x23.y : -INFINITY;
            am = __fadd2_rn(am, make_float2(ex2(x01.x), ex2(x01.y)));
            ap = __fadd2_rn(ap, (c4 & 1) ? exp2_fma2(x23) : make_float2(ex2(x23.x), ex2(x23.y)));
        }
    }
}

// Next visible column block after b in a 256-bit mask (-1: none).
__device__ __forceinline__ int next_visible(const uint32_t *vmask, int b) {
    for (int x = b + 1; x < kMaxBlocks; ++x) {
        const uint32_t w = vmask[x >> 5] >> (x & 31);
        if (w == 0u) {
            x |= 31;
            continue;
        }
        return x + __ffs(w) - 1;
    }
    return -1;
}

// ---------------------------------------------------------------- shared memory plan
template <int D>
struct Plan {
    static constexpr int kChunks = D / 64;                       // 128-byte K chunks
    static constexpr int kABytes = kTileKeys * D * 2;           // whole K tile
    static constexpr int kBBytes = kCols * D * 2;                // one Q block
    static constexpr int kStages = D == 128 ? 2 : 4;
    static constexpr int kOffA = 0;                              // two K tiles
    static constexpr int kOffB = 2 * kABytes;
    static constexpr int kOffItems = kOffB + kStages * kBBytes;
    static constexpr int kOffCtrl = kOffItems + kMeta * (int)sizeof(Item);
    static constexpr int kBytes = kOffCtrl + (int)sizeof(Ctrl) + 1024;  // + alignment slack
    static_assert(kBytes <= 232448, "shared memory plan exceeds 227 KB per CTA");
};

// ---------------------------------------------------------------- the kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q, TcArgs a) {
    using PL = Plan<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + PL::kOffA;
    uint8_t *sB = smem + PL::kOffB;
    Item *items = reinterpret_cast<Item *>(smem + PL::kOffItems);
    Ctrl &ctl = *reinterpret_cast<Ctrl *>(smem + PL::kOffCtrl);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const CacheView &c = a.c;

    if (warp == 2 && (int64_t)blockIdx.x < a.total_tiles) {
        // warm L2 with what the first tile's decode reads (the CTA's first tile has index blockIdx.x): its row
        // length, block-table entries and slot positions, and the sequence's query count and positions
        const int RPS0 = c.num_layers * c.num_kv_heads;
        const int64_t tid = blockIdx.x, rr = tid % RPS0, rest = tid / RPS0;
        const int t = (int)(rest % a.tiles_per_row), seq = (int)(rest / a.tiles_per_row);
        const int64_t row = (int64_t)seq * RPS0 + rr;
        const int32_t *line =
            lane == 0 ? c.row_len + row
                      : (lane == 1 ? c.block_table + row * c.max_pages_per_row + min(t * kPagesPerTile, c.max_pages_per_row - 1)
                                   : a.q.num_q + seq);
        if (lane < 3) asm volatile("prefetch.global.L2 [%0];" ::"l"(line));
        const int32_t *sp = c.slot_pos + row * c.max_slots + (int64_t)t * kTileKeys;
        const int nk = (int)min((int64_t)kTileKeys, c.max_slots - (int64_t)t * kTileKeys);
        if (lane * 32 < nk) asm volatile("prefetch.global.L2 [%0];" ::"l"(sp + lane * 32));
        const int32_t *qp = a.q.q_pos + (int64_t)seq * a.q.max_q;
        for (int j = lane * 32; j < a.q.max_q; j += 32 * 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(qp + j));
    }
    // The first tile's sequence: the q_pos range of each of its query blocks, computed by the whole CTA (one
    // load per thread and query) so that the decoder starts with it instead of gathering it alone.
    int seq0 = -1, nq0 = 0;
    if ((int64_t)blockIdx.x < a.total_tiles) {
        seq0 = (int)(((int64_t)blockIdx.x / (c.num_layers * c.num_kv_heads)) / a.tiles_per_row);
        nq0 = min(a.q.num_q[seq0], a.q.max_q);
        for (int b = threadIdx.x; b < (nq0 + a.nqb - 1) / a.nqb; b += kThreads) {
            ctl.blk_qmin[0][b] = INT32_MAX;
            ctl.blk_qmax[0][b] = INT32_MIN;
        }
    }
    __syncthreads();
    if (seq0 >= 0) {
        const int32_t *qrow = a.q.q_pos + (int64_t)seq0 * a.q.max_q;
        for (int j = threadIdx.x; j < nq0; j += kThreads) {
            const int p = qrow[j];
            atomicMin(&ctl.blk_qmin[0][j / a.nqb], p);
            atomicMax(&ctl.blk_qmax[0][j / a.nqb], p);
        }
    }
    // zero the operand buffers once so rows no load ever fills hold finite values
    for (int i = threadIdx.x; i < (2 * PL::kABytes + PL::kStages * PL::kBBytes) / 16; i += kThreads)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < PL::kStages; ++s) {
            mbar_init(&ctl.q_full[s], 1);
            mbar_init(&ctl.q_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.a_full[b], 1);
            mbar_init(&ctl.a_empty[b], 1);
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], kEpiWarps);
            mbar_init(&ctl.part_full[b], kEpiWarps / 2);
        }
        for (int k = 0; k < kMeta; ++k) {
            mbar_init(&ctl.m_full[k], 1);
            mbar_init(&ctl.m_empty[k], kEpiWarps);
        }
        for (int k = 0; k < kTiles; ++k) {
            mbar_init(&ctl.t_full[k], 1);
            mbar_init(&ctl.t_empty[k], 2);  // TMA and MMA warps
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

    const int G = a.q.group, Hq = a.q.num_q_heads, nqb = a.nqb;
    const int RPS = c.num_layers * c.num_kv_heads;

    if (warp == 0) {
        // ============================== TMA loads ==============================
        // Follows the tile ring: per tile, the K tile into the free A buffer, then the Q block of every visible
        // column block into the stage ring, in the order the MMA warp consumes them.
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_q)) : "memory");
        uint32_t qs = 0, qph = 0, tk = 0, tph = 0;
        uint32_t ta = 0;  // K tiles loaded so far: buffer ta & 1, use (ta >> 1) of that buffer
        const uint32_t a_tx_page = 16 * 128;                 // one 16-row, 128-byte box
        const uint32_t q_tx = (uint32_t)(G * nqb) * 128u;    // one Q box per 64-column chunk
        bool ok = true;
        for (;;) {
            if (!mbar_wait(&ctl.t_full[tk], tph, ctl, a.status, -1)) { ok = false; break; }
            const TileRec &R = ctl.trec[tk];
            const int row = R.row;
            if (row < 0) break;
            const int zq = R.seq * c.num_layers + R.layer, hq0 = R.kvh * G, first_vis = R.first_vis;
            const unsigned okmask = R.okmask;
            const int my_page = lane < kPagesPerTile ? R.page[lane] : -1;
            // K tile into the free buffer: one box per (page, 64-column chunk)
            const uint32_t abuf = ta & 1;
            if (!mbar_wait(&ctl.a_empty[abuf], ((ta >> 1) & 1) ^ 1, ctl, a.status, row)) { ok = false; break; }
            ++ta;
            if (lane == 0) mbar_expect_tx(&ctl.a_full[abuf], (uint32_t)__popc(okmask) * a_tx_page * PL::kChunks);
            __syncwarp();
            if (my_page >= 0) {
                const int half = lane >> 3, r0 = (lane & 7) * 16;
#pragma unroll
                for (int kc = 0; kc < PL::kChunks; ++kc) {
                    const uint32_t dst =
                        smem_u32(sA + abuf * PL::kABytes + kc * (kTileKeys * 128) + half * (128 * 128) + r0 * 128);
                    tma_load_2d(dst, &tmap_k, &ctl.a_full[abuf], kc * 64, my_page * 16);
                }
            }
            // Q blocks of the visible column blocks
            for (int b = first_vis; b >= 0; b = next_visible(R.vmask, b)) {
                if (!mbar_wait(&ctl.q_empty[qs], qph ^ 1, ctl, a.status, row)) { ok = false; break; }
                if (lane == 0) {
                    mbar_expect_tx(&ctl.q_full[qs], q_tx * PL::kChunks);
#pragma unroll
                    for (int kc = 0; kc < PL::kChunks; ++kc) {
                        const uint32_t dst = smem_u32(sB + qs * PL::kBBytes + kc * (kCols * 128));
                        tma_load_4d(dst, &tmap_q, &ctl.q_full[qs], kc * 64, b * nqb, hq0, zq);
                    }
                }
                __syncwarp();
                if (++qs == PL::kStages) { qs = 0; qph ^= 1; }
            }
            if (!ok) break;
            if (lane == 0) mbar_arrive(&ctl.t_empty[tk]);
            if (++tk == kTiles) { tk = 0; tph ^= 1; }
        }
        if (!ok || ctl.abort) {
            // drain our own copies before the CTA can exit: every issued TMA phase completes
            for (int s = 0; s < PL::kStages; ++s) {
                const uint64_t t0 = now_ns();
                while (!mbar_test(&ctl.q_full[s], (qph ^ (s < (int)qs ? 0u : 1u)) & 1u) && now_ns() - t0 < kTimeoutNs) {}
            }
            for (uint32_t b = 0; b < 2; ++b) {
                const uint32_t fills = (ta + 1 - b) / 2;  // loads that went to buffer b
                if (fills == 0) continue;
                const uint64_t t0 = now_ns();
                while (!mbar_test(&ctl.a_full[b], (fills - 1) & 1) && now_ns() - t0 < kTimeoutNs) {}
            }
        }
    } else if (warp == 2) {
        // ============================== tiles and column data ==============================
        // Decodes each tile one tile ahead (row length, block-table entries, slot positions, visible column
        // blocks) and hands it to the TMA warp through the tile ring; copies every visible block's raw column
        // data a block ahead with cp.async; converts it and publishes one metadata item per block.
        uint32_t mk = 0, mph = 0, tk = 0, tph = 0;
        // q_pos ranges of a sequence's blocks live in one of two buffers: the tile being produced and the one
        // decoded ahead of it may belong to different sequences
        int cur_seq = seq0, nq = nq0, nblk = seq0 >= 0 ? (nq0 + nqb - 1) / nqb : 0, sbuf = 0;
        bool ok = true;
        const int mp = c.max_pages_per_row;
        const int64_t ms = c.max_slots;
        // Raw loads of a tile (row length, its block-table entries and slot positions), issued a whole tile
        // before they are used; nothing branches on a loaded value until then.
        struct TileRaw {
            int64_t tid;
            int n, page, kp[8];
        };
        auto issue_tile = [&](int64_t tid, TileRaw &r) {
            r.tid = tid;
            if (tid >= a.total_tiles) return;
            const int64_t rr = tid % RPS, rest = tid / RPS;
            const int t = (int)(rest % a.tiles_per_row), seq = (int)(rest / a.tiles_per_row);
            const int64_t row = (int64_t)seq * RPS + rr;
            r.n = c.row_len[row];
            r.page = c.block_table[row * mp + min(t * kPagesPerTile + (lane & 15), mp - 1)];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                r.kp[i] = c.slot_pos[row * ms + min((int64_t)t * kTileKeys + i * 32 + lane, ms - 1)];
        };
        // Decode a tile (waits for its raw loads) into T (shared) and key staging buffer `parity`; a tile with a visible
        // block also goes to the TMA warp.  Returns false for a tile with no keys (or on abort, with ok cleared).
        auto make_tile = [&](const TileRaw &r, int parity, Tile &T) -> bool {
            if (r.tid >= a.total_tiles) return false;
            const int64_t rr = r.tid % RPS, rest = r.tid / RPS;
            const int t = (int)(rest % a.tiles_per_row);
            const int seq = (int)(rest / a.tiles_per_row);
            const int row = seq * RPS + (int)rr;
            const int n = r.n;
            if (n < 0 || n > ms) {
                if (t == 0 && lane == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
                return false;
            }
            const int k0 = t * kTileKeys;
            if (k0 >= n) return false;
            const int n_keys = min(kTileKeys, n - k0);
            if (seq != cur_seq) {
                cur_seq = seq;
                sbuf ^= 1;
                nq = min(a.q.num_q[seq], a.q.max_q);
                nblk = (nq + nqb - 1) / nqb;
                for (int b = lane; b < nblk; b += 32) {
                    ctl.blk_qmin[sbuf][b] = INT32_MAX;
                    ctl.blk_qmax[sbuf][b] = INT32_MIN;
                }
                __syncwarp();
                // q_pos range of every block: coalesced loads, four in flight per lane, shared-memory atomics
                const int32_t *qrow = a.q.q_pos + (int64_t)seq * a.q.max_q;
                for (int j0 = 0; j0 < nq; j0 += 128) {
                    int pv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = j0 + u * 32 + lane;
                        pv[u] = j < nq ? qrow[j] : 0;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = j0 + u * 32 + lane;
                        if (j < nq) {
                            atomicMin(&ctl.blk_qmin[sbuf][j / nqb], pv[u]);
                            atomicMax(&ctl.blk_qmax[sbuf][j / nqb], pv[u]);
                        }
                    }
                }
                __syncwarp();
            }
            bool page_ok = false;
            if (lane < kPagesPerTile && k0 + lane * 16 < n) {
                page_ok = r.page >= 0 && r.page < c.num_pages;
                if (!page_ok) report(a.status, KVC_DEV_BAD_PAGE, row);
            }
            const unsigned okmask = __ballot_sync(0xffffffffu, page_ok);
            int kmin = INT32_MAX;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int key = i * 32 + lane;
                const bool v = key < n_keys && ((okmask >> (key >> 4)) & 1u);
                const int kp = v ? r.kp[i] : INT32_MAX;
                ctl.kstage[parity][key] = kp;
                if (v) kmin = min(kmin, kp);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            // visible blocks: some query at or after the tile's first key position
            int first_vis = -1, last_vis = -1;
#pragma unroll
            for (int w = 0; w < kMaxBlocks / 32; ++w) {
                const int b = w * 32 + lane;
                const bool v = b < nblk && ctl.blk_qmax[sbuf][b] >= kmin;
                const unsigned m = __ballot_sync(0xffffffffu, v);
                if (lane == 0) ctl.vstage[parity][w] = m;
                if (m) {
                    if (first_vis < 0) first_vis = w * 32 + __ffs(m) - 1;
                    last_vis = w * 32 + 31 - __clz(m);
                }
            }
            if (lane < 8) {
                // readable keys lane*32 .. lane*32+31: below n_keys, in one of the lane's two pages that loaded
                const int k0l = lane * 32;
                const uint32_t keym =
                    n_keys >= k0l + 32 ? 0xFFFFFFFFu : (n_keys <= k0l ? 0u : ((1u << (n_keys - k0l)) - 1u));
                const uint32_t pg = (okmask >> (2 * lane)) & 3u;
                const uint32_t pagem = ((pg & 1u) ? 0x0000FFFFu : 0u) | ((pg & 2u) ? 0xFFFF0000u : 0u);
                ctl.kvstage[parity][lane] = keym & pagem;
            }
            const int layer = (int)(rr / c.num_kv_heads), kvh = (int)(rr % c.num_kv_heads);
            if (lane == 0) {
                T.row = row;
                T.t = t;
                T.n_keys = n_keys;
                T.first_vis = first_vis;
                T.last_vis = last_vis;
                T.nq = nq;
                T.sbuf = sbuf;
                T.lrow = a.q.lse + ((int64_t)(seq * c.num_layers + layer) * Hq + kvh * G) * a.q.max_q;
                T.prow = a.q.q_pos + (int64_t)seq * a.q.max_q;
            }
            __syncwarp();
            if (first_vis >= 0) {
                if (!mbar_wait(&ctl.t_empty[tk], tph ^ 1, ctl, a.status, row)) {
                    ok = false;
                    return false;
                }
                TileRec &R = ctl.trec[tk];
                if (lane < kPagesPerTile) R.page[lane] = page_ok ? r.page : -1;
                if (lane < kMaxBlocks / 32) R.vmask[lane] = ctl.vstage[parity][lane];
                if (lane == 0) {
                    R.row = row;
                    R.seq = seq;
                    R.layer = layer;
                    R.kvh = kvh;
                    R.okmask = okmask;
                    R.first_vis = first_vis;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.t_full[tk]);
                if (++tk == kTiles) { tk = 0; tph ^= 1; }
            }
            return true;
        };
        // Column data (lse, q_pos) of a block, copied asynchronously into a staging slot of shared memory
        // (cp.async: no register waits on the copies); one commit group per call, possibly empty.
        // Slots in use at any time: the current block's, the next tile's first block's, and the one being
        // filled for the next block of this tile; a new slot is any other of the four.
        auto pick_slot = [](uint32_t x, uint32_t y) -> uint32_t {
            uint32_t s = 0;
            while (s == x || s == y) ++s;
            return s;
        };
        auto issue_cols = [&](const Tile &f, bool valid, int b, uint32_t slot) -> uint32_t {
            if (valid) {
                const int mq = a.q.max_q, j0 = b * nqb;
                ColStage &cs = ctl.colstage[slot];
                if (a.vec) {
                    // 16-byte pieces: lse in column order (head-major), then q_pos; pieces past max_q read nothing
                    if (lane < G * nqb / 4) {
                        const int col = lane * 4, g = col / nqb, j = j0 + col % nqb;
                        const int avail = max(0, min(4, mq - j)) * 4;
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(&cs.lse[col])),
                                     "l"(f.lrow + (int64_t)g * mq + (avail ? j : 0)), "r"(avail)
                                     : "memory");
                    }
                    if (lane < nqb / 4) {
                        const int j = j0 + lane * 4;
                        const int avail = max(0, min(4, mq - j)) * 4;
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(&cs.qpos[lane * 4])),
                                     "l"(f.prow + (avail ? j : 0)), "r"(avail)
                                     : "memory");
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int col = u * 32 + lane;
                        if (col < G * nqb) {
                            const int g = col / nqb, j = min(j0 + col % nqb, mq - 1);
                            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&cs.lse[col])),
                                         "l"(f.lrow + (int64_t)g * mq + j)
                                         : "memory");
                        }
                        if (col < nqb) {
                            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&cs.qpos[col])),
                                         "l"(f.prow + min(j0 + col, mq - 1))
                                         : "memory");
                        }
                    }
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            return slot;
        };
        // This lane's four columns of every block: 4*lane .. 4*lane+3, query index within the block (or -1
        // for a column past the group's G*nqb).  With nqb % 4 == 0 the four share one head.
        int cjl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int col = 4 * lane + i;
            cjl[i] = col < G * nqb ? col % nqb : -1;
        }
        const bool q4 = (nqb & 3) == 0;
        auto fill_tile_part = [&](Item &it, int parity) {
#pragma unroll
            for (int i = 0; i < 8; ++i) it.kpos[i * 32 + lane] = ctl.kstage[parity][i * 32 + lane];
            if (lane < 8) it.kvalid[lane] = ctl.kvstage[parity][lane];
        };

        // Tile order: round k takes tiles k * grid .. k * grid + grid - 1, CTA b the b-th of them in even rounds
        // and the (grid - 1 - b)-th in odd rounds, so that the costly and the cheap ends of the order (under a
        // causal mask, early positions see more query blocks) share out across CTAs.
        int64_t round_next = 0;
        auto next_tid = [&]() -> int64_t {
            const int64_t k = round_next++;
            return k * gridDim.x + ((k & 1) ? (int64_t)(gridDim.x - 1 - blockIdx.x) : (int64_t)blockIdx.x);
        };
        TileRaw raw;
        Tile cur{};
        Tile &nxt = ctl.tnext;
        uint32_t cslot = 0, nslot = 0;  // staging slots of the current block and of the next tile's first block
        int par = 0;
        int64_t tid_next = next_tid();
        // find the first tile with keys
        bool have = false;
        while (ok && !have && tid_next < a.total_tiles) {
            issue_tile(tid_next, raw);
            tid_next = next_tid();
            have = make_tile(raw, par, nxt);
        }
        nslot = issue_cols(nxt, ok && have && nxt.first_vis >= 0, nxt.first_vis, 0);
        if (tid_next < a.total_tiles) issue_tile(tid_next, raw);
        // Decode the following tile (its loads were issued a tile ago) and copy its first block's columns; done
        // once the current tile's first item is out, so that the first item does not wait for it.
        auto decode_next = [&](uint32_t busy) {
            par ^= 1;
            have = false;
            while (ok && !have && tid_next < a.total_tiles) {
                const TileRaw r = raw;
                tid_next = next_tid();
                if (tid_next < a.total_tiles) issue_tile(tid_next, raw);
                have = make_tile(r, par, nxt);
            }
            nslot = issue_cols(nxt, ok && have && nxt.first_vis >= 0, nxt.first_vis, pick_slot(busy, busy));
        };
        while (ok && have) {
            cur = nxt;
            cslot = nslot;
            const int cpar = par;
            if (cur.first_vis < 0) {
                if (!mbar_wait(&ctl.m_empty[mk], mph ^ 1, ctl, a.status, cur.row)) { ok = false; break; }
                Item &it = items[mk];
                fill_tile_part(it, cpar);
                if (lane == 0) {
                    *reinterpret_cast<int4 *>(&it.row) = make_int4(cur.row, cur.t, -1, kFirst | kLast);
                    *reinterpret_cast<int4 *>(&it.n_keys) = make_int4(cur.n_keys, 0, INT32_MAX, INT32_MIN);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.m_full[mk]);
                if (++mk == kMeta) { mk = 0; mph ^= 1; }
                decode_next(cslot);
                continue;
            }
            bool decoded = false, after_decode = false;
            for (int b = cur.first_vis; b >= 0;) {
                const int bn = next_visible(ctl.vstage[cpar], b);
                const uint32_t bslot = issue_cols(cur, bn >= 0, bn, pick_slot(cslot, decoded ? nslot : cslot));
                // metadata item (the column data was copied a block earlier)
                if (!mbar_wait(&ctl.m_empty[mk], mph ^ 1, ctl, a.status, cur.row)) { ok = false; break; }
                Item &it = items[mk];
                const int flags = (b == cur.first_vis ? kFirst : 0) | (b == cur.last_vis ? kLast : 0);
                if (flags & kFirst) fill_tile_part(it, cpar);
                const int vq = min(nqb, cur.nq - b * nqb);
                // this block's staged columns have landed; the group just issued may stay in flight, and right after
                // the next tile's decode so may the next tile's first block (committed between the two)
                if (after_decode)
                    asm volatile("cp.async.wait_group 2;" ::: "memory");
                else
                    asm volatile("cp.async.wait_group 1;" ::: "memory");
                after_decode = false;
                __syncwarp();
                {
                    // four columns per lane: one 16-byte read of the raw lse, converted, one 16-byte write
                    const ColStage &cs = ctl.colstage[cslot];
                    const float4 lr = *reinterpret_cast<const float4 *>(&cs.lse[4 * lane]);
                    int4 qv;
                    if (q4 && cjl[0] >= 0) {
                        qv = *reinterpret_cast<const int4 *>(&cs.qpos[cjl[0]]);
                    } else {
                        qv.x = cjl[0] >= 0 ? cs.qpos[cjl[0]] : 0;
                        qv.y = cjl[1] >= 0 ? cs.qpos[cjl[1]] : 0;
                        qv.z = cjl[2] >= 0 ? cs.qpos[cjl[2]] : 0;
                        qv.w = cjl[3] >= 0 ? cs.qpos[cjl[3]] : 0;
                    }
                    const float lv[4] = {lr.x, lr.y, lr.z, lr.w};
                    const int pv[4] = {qv.x, qv.y, qv.z, qv.w};
                    float nl[4];
                    int qq[4];
                    bool any = false;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        nl[i] = -INFINITY;
                        qq[i] = INT32_MIN;
                        if (cjl[i] >= 0 && cjl[i] < vq) {
                            const float l = lv[i];
                            if (l == -INFINITY) {
                                // a column that saw no key contributes nothing
                            } else if (!is_finite(l)) {
                                report(a.status, KVC_DEV_NONFINITE, cur.row);
                            } else {
                                nl[i] = -l * 1.4426950408889634f;
                                qq[i] = pv[i];
                                any = true;
                            }
                        }
                    }
                    *reinterpret_cast<float4 *>(&it.nL[4 * lane]) = make_float4(nl[0], nl[1], nl[2], nl[3]);
                    *reinterpret_cast<int4 *>(&it.qp[4 * lane]) = make_int4(qq[0], qq[1], qq[2], qq[3]);
                    const unsigned bal = __ballot_sync(0xffffffffu, any);
                    if (lane == 0) {
                        const int chunks = ((bal & 0xFFu) ? 1 : 0) | ((bal & 0xFF00u) ? 2 : 0) |
                                           ((bal & 0xFF0000u) ? 4 : 0) | ((bal & 0xFF000000u) ? 8 : 0);
                        *reinterpret_cast<int4 *>(&it.row) = make_int4(cur.row, cur.t, b, flags);
                        *reinterpret_cast<int4 *>(&it.n_keys) =
                            make_int4(cur.n_keys, chunks, ctl.blk_qmin[cur.sbuf][b], ctl.blk_qmax[cur.sbuf][b]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.m_full[mk]);
                if (++mk == kMeta) { mk = 0; mph ^= 1; }
                if (!decoded) {
                    decode_next(bslot);
                    if (!ok) break;
                    decoded = after_decode = true;
                }
                b = bn;
                cslot = bslot;
            }
        }
        // end-of-work markers: for the MMA and epilogue warps, and for the TMA warp
        if (ok && mbar_wait(&ctl.m_empty[mk], mph ^ 1, ctl, a.status, -1)) {
            if (lane == 0) {
                items[mk].row = -1;
                mbar_arrive(&ctl.m_full[mk]);
            }
        }
        if (ok && mbar_wait(&ctl.t_empty[tk], tph ^ 1, ctl, a.status, -1)) {
            if (lane == 0) {
                ctl.trec[tk].row = -1;
                mbar_arrive(&ctl.t_full[tk]);
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // no copy into shared memory outlives the CTA
    } else if (warp == 1) {
        // ============================== MMA issuer ==============================
        // Follows the tile ring like the TMA warp: per tile the K buffer, per visible block the Q stage and an
        // accumulator buffer; two M=128 x N=128 x K=D products per block, one thread issuing.
        uint32_t qs = 0, qph = 0, tk = 0, tph = 0, ab = 0, abph = 0;
        uint32_t tm = 0;  // K tiles consumed so far (same order as the TMA warp's loads)
        bool issued = false;
        const uint32_t a_lo0 = desc_lo(smem_u32(sA)), b_lo0 = desc_lo(smem_u32(sB));
        for (;;) {
            if (!mbar_wait(&ctl.t_full[tk], tph, ctl, a.status, -1)) break;
            const TileRec &R = ctl.trec[tk];
            const int row = R.row;
            if (row < 0) break;
            const uint32_t abuf = tm & 1;
            if (!mbar_wait(&ctl.a_full[abuf], (tm >> 1) & 1, ctl, a.status, row)) break;
            const uint32_t a_lo = a_lo0 + ((abuf * PL::kABytes) >> 4);
            bool ok = true;
            for (int b = R.first_vis; b >= 0;) {
                const int bn = next_visible(R.vmask, b);
                if (!mbar_wait(&ctl.q_full[qs], qph, ctl, a.status, row)) { ok = false; break; }
                if (!mbar_wait(&ctl.acc_empty[ab], abph ^ 1, ctl, a.status, row)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t b_lo = b_lo0 + ((qs * PL::kBBytes) >> 4);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t d = tmem + ab * 256 + h * kCols;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t ao = (uint32_t)(((kk >> 2) * (kTileKeys * 128) + h * (128 * 128) + (kk & 3) * 32) >> 4);
                            const uint32_t bo = (uint32_t)(((kk >> 2) * (kCols * 128) + (kk & 3) * 32) >> 4);
                            if (kk == 0)
                                mma_bf16<false>(d, a_lo + ao, b_lo + bo);
                            else
                                mma_bf16<true>(d, a_lo + ao, b_lo + bo);
                        }
                    }
                    mma_commit(&ctl.q_empty[qs]);
                    mma_commit(&ctl.acc_full[ab]);
                    if (bn < 0) mma_commit(&ctl.a_empty[abuf]);
                }
                issued = true;
                __syncwarp();
                if (++qs == PL::kStages) { qs = 0; qph ^= 1; }
                if (++ab == 2) { ab = 0; abph ^= 1; }
                b = bn;
            }
            if (!ok) break;
            ++tm;
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.t_empty[tk]);
            if (++tk == kTiles) { tk = 0; tph ^= 1; }
        }
        // all MMAs issued by this thread are complete before TMEM is released
        if (issued) {
            if (lane == 0) mma_commit(&ctl.drain);
            __syncwarp();
            const uint64_t t0 = now_ns();
            while (!mbar_test(&ctl.drain, 0) && now_ns() - t0 < kTimeoutNs) {}
        }
    } else if (warp >= 3) {
        // ============================== epilogue ==============================
        // 16 warps: (TMEM lane quadrant = warp % 4, key half, column half); the two column halves of a key
        // are added through shared memory at the end of each tile.
        const int e = warp - 3;
        const int quad = warp & 3, half = (e >> 2) & 1, colh = e >> 3;
        const int key = half * 128 + quad * 32 + lane;  // key within the tile = TMEM lane of its half
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        uint32_t mk = 0, mph = 0, ab = 0, abph = 0, tcount = 0;
        float2 am = make_float2(0.f, 0.f), ap = make_float2(0.f, 0.f);
        int kpos = INT32_MAX, wkmin = INT32_MAX, wkmax = INT32_MIN;
        bool kv = false;
        const float sc = a.scale_log2e;
        for (;;) {
            if (!mbar_wait(&ctl.m_full[mk], mph, ctl, a.status, -1)) break;
            const Item &it = items[mk];
            const int row = it.row;
            if (row < 0) break;
            const int flags = it.flags, blk = it.blk;
            if (flags & kFirst) {
                am = ap = make_float2(0.f, 0.f);
                kv = (it.kvalid[key >> 5] >> (key & 31)) & 1u;
                kpos = it.kpos[key];
                int mn = kv ? kpos : INT32_MAX, mx = kv ? kpos : INT32_MIN;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
                wkmin = mn;
                wkmax = mx;
            }
            float *dst = a.scores + (int64_t)row * c.max_slots + (int64_t)it.tile * kTileKeys + key;
            if (blk >= 0) {
                if (!mbar_wait(&ctl.acc_full[ab], abph, ctl, a.status, row)) break;
                tc_fence_after();
                const int4 hd = *reinterpret_cast<const int4 *>(&it.n_keys);  // n_keys, chunks, qmin, qmax
                const uint32_t tbase = tmem + lane_addr + ab * 256 + half * kCols + colh * 64;
                const int ch0 = colh * 2, ch1 = ch0 + 1;
                // a chunk is skipped when it holds no present column or no key of this warp sees any query of
                // the block; when every query of the block sees every key of the warp, no causal select
                const bool sees = wkmax != INT32_MIN && hd.w >= wkmin;
                const bool fast = hd.z >= wkmax;
                // 16-column TMEM loads, double-buffered: the next one is in flight while the current is summed
                const bool do0 = sees && ((hd.y >> ch0) & 1), do1 = sees && ((hd.y >> ch1) & 1);
                const float *nL = it.nL + colh * 64;
                const int32_t *qp = it.qp + colh * 64;
                uint32_t ra[16], rb[16];
                if (do0 && do1) {
                    tmem_ld16(tbase, ra);
                    tmem_wait16(ra);
                    tmem_ld16(tbase + 16, rb);
                    epi16(ra, nL, qp, kpos, sc, fast, am, ap);
                    tmem_wait16(rb);
                    tmem_ld16(tbase + 32, ra);
                    epi16(rb, nL + 16, qp + 16, kpos, sc, fast, am, ap);
                    tmem_wait16(ra);
                    tmem_ld16(tbase + 48, rb);
                    epi16(ra, nL + 32, qp + 32, kpos, sc, fast, am, ap);
                    tmem_wait16(rb);
                    epi16(rb, nL + 48, qp + 48, kpos, sc, fast, am, ap);
                } else if (do0 || do1) {
                    const int o = do0 ? 0 : 32;
                    tmem_ld16(tbase + o, ra);
                    tmem_wait16(ra);
                    tmem_ld16(tbase + o + 16, rb);
                    epi16(ra, nL + o, qp + o, kpos, sc, fast, am, ap);
                    tmem_wait16(rb);
                    epi16(rb, nL + o + 16, qp + o + 16, kpos, sc, fast, am, ap);
                }
                tc_fence_before();
                if (flags & kLast) {
                    // add the column halves (before the accumulator is released, see below)
                    const uint32_t p = tcount & 1, ph = (tcount >> 1) & 1;
                    ++tcount;
                    if (colh == 1) {
                        ctl.part[p][key] = (am.x + am.y) + (ap.x + ap.y);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl.part_full[p]);
                    } else {
                        if (!mbar_wait(&ctl.part_full[p], ph, ctl, a.status, row)) break;
                        if (kv) {
                            const float v = ((am.x + am.y) + (ap.x + ap.y)) + ctl.part[p][key];
                            *dst = a.accumulate ? *dst + v : v;
                        }
                    }
                }
                // Releasing the buffer after the column-half exchange keeps part[p] from being rewritten
                // before it is read: its next writer must first obtain an accumulator this warp released.
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.acc_empty[ab]);
                if (++ab == 2) { ab = 0; abph ^= 1; }
            } else if ((flags & kLast) && colh == 0 && kv) {
                if (!a.accumulate) *dst = 0.f;  // no query sees this tile
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.m_empty[mk]);
            if (++mk == kMeta) { mk = 0; mph ^= 1; }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

// ---------------------------------------------------------------- host side

template <int D>
cudaError_t launch_t(const CacheView &c, const QueryView &q, float *scores, bool accumulate, int32_t *status,
                     cudaStream_t stream, char *err, size_t errlen) {
    using PL = Plan<D>;
    if (!tmap_encoder()) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled unavailable");
        return cudaErrorNotSupported;
    }
    const int G = q.group;
    const int nqb = kCols / G;
    if ((q.max_q + nqb - 1) / nqb > kMaxBlocks) {
        snprintf(err, errlen, "query set too large for one pass: max_q %d > %d", q.max_q, kMaxBlocks * nqb);
        return cudaErrorInvalidValue;
    }
    CUtensorMap tk, tq;
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)c.num_pages * 16};
        cuuint64_t strides[1] = {(cuuint64_t)D * 2};
        cuuint32_t box[2] = {64, 16};
        CUresult r = tmap_bf16(kTmapScoreK, &tk, 2, c.k_pool, dims, strides, box);
        if (r != CUDA_SUCCESS) {
            snprintf(err, errlen, "K tensor map encode failed (%d)", (int)r);
            return cudaErrorInvalidValue;
        }
    }
    {
        // dimensions (D, query, head, seq*layer): a box lands head-major, column n = g * nqb + query
        cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)q.max_q, (cuuint64_t)q.num_q_heads,
                              (cuuint64_t)c.num_seqs * c.num_layers};
        cuuint64_t strides[3] = {(cuuint64_t)q.num_q_heads * D * 2, (cuuint64_t)D * 2,
                                 (cuuint64_t)q.max_q * q.num_q_heads * D * 2};
        cuuint32_t box[4] = {64, (cuuint32_t)nqb, (cuuint32_t)G, 1};
        CUresult r = tmap_bf16(kTmapScoreQ, &tq, 4, q.q, dims, strides, box);
        if (r != CUDA_SUCCESS) {
            snprintf(err, errlen, "Q tensor map encode failed (%d)", (int)r);
            return cudaErrorInvalidValue;
        }
    }
    TcArgs args;
    args.c = c;
    args.q = q;
    args.scores = scores;
    args.status = status;
    args.accumulate = accumulate ? 1 : 0;
    args.vec = ((reinterpret_cast<uintptr_t>(q.lse) | reinterpret_cast<uintptr_t>(q.q_pos)) & 15) == 0 &&
               q.max_q % 4 == 0 && nqb % 4 == 0;
    args.nqb = nqb;
    args.tiles_per_row = (int)((c.max_slots + kTileKeys - 1) / kTileKeys);
    args.total_tiles = (int64_t)c.rows * args.tiles_per_row;
    args.scale_log2e = (float)(1.4426950408889634 / std::sqrt((double)D));
    const int sms = device_sms();
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)score_tc_kernel<D>, PL::kBytes, smem_set);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(sms, args.total_tiles);
    score_tc_kernel<D><<<grid, kThreads, PL::kBytes, stream>>>(tk, tq, args);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_tc(const CacheView &c, const QueryView &q, float *scores, bool accumulate, int32_t *status,
                            cudaStream_t stream, char *err, size_t errlen) {
    if (c.head_dim == 64) return launch_t<64>(c, q, scores, accumulate, status, stream, err, errlen);
    return launch_t<128>(c, q, scores, accumulate, status, stream, err, errlen);
}

}  // namespace kvc
