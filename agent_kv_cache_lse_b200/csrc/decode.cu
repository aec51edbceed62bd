// One decode step of paged attention with the eviction scores folded in.
//
// "ActKV Dissected", Component 3: the softmax log-sum-exp is a byproduct of paged attention,
// so the current query's attention probabilities are its logits minus the LSE, with no gather
// of the attention matrix and no recompute.  Here the decode kernel does it itself.  For each
// row (sequence, layer, KV head), the G query heads of its group and the row's keys at or
// before the query's position:
//   l[g, i] = q_g . k_i / sqrt(D),  lse[g] = log sum_i exp(l[g, i]),
//   out[g] = sum_i exp(l[g, i] - lse[g]) v_i,  scores[i] (+)= sum_g exp(l[g, i] - lse[g]).
//
// One cluster of C CTAs per row; each CTA owns a contiguous run of the row's chunks (CH slots of
// one page, CH the largest divisor of the page size up to 16).  In a CTA of eight warps:
//   * warp w takes chunks w, w + 8, ...  It streams its own chunks' K and V bytes into a private
//     ring of RW shared-memory stages with 16-byte cp.async copies (every lane issues its share;
//     the block-table entries come 32 chunks at a time, one per lane), RW - 1 chunks ahead of the
//     one it works on.  Bulk copies (cp.async.bulk) of one 4 KB page each were measured to cap a
//     B200 SM near 15 GB/s (the copy engine's per-copy time, not the ring depth, sets the rate),
//     so every warp issues its own loads instead;
//   * a lane owns 8 elements of D of one key (KW = 32 / (D/8) keys per step) and holds the
//     group's query slice in registers; the warp forms the chunk's logits (base-2 domain, causal
//     mask from the slot positions, which are staged in shared memory once), writes them to a
//     shared-memory logits buffer, and folds the chunk into its running maximum, sum and output
//     (online softmax: a new maximum rescales the sum and output once per chunk);
//   * the warps' (max, sum, output) merge in warp order, then the cluster's in rank order through
//     distributed shared memory; the leader writes out = O / S and lse = (M + log2 S) ln 2, and
//     every CTA adds sum_g 2^(l - M_g) / S_g to its slots' scores from the logits it kept.
// Every sum runs in a fixed order, so results repeat bit for bit from run to run.  The kernel has
// no spin-waits: cp.async groups always complete, and the cluster barriers are taken by all CTAs.
//
// Where the lanes' logits are reduce-scattered (two lanes per key) and the slot positions and scores
// can be copied 16 bytes at a time, the kept logits leave shared memory for tensor memory (TMEM, which
// this kernel has no other use for): each lane stores its logits of a chunk into its own TMEM lane
// (tcgen05.st), and each chunk's stage also carries the chunk's slot positions and, when accumulating,
// its old scores (stored to TMEM beside the logits).  Shared memory then holds only the K/V stages, so
// every warp keeps two chunks in flight instead of one, and the final scores need no global reads.
//
// With bf16 K/V and 16-slot chunks, a chunk's two contractions run on the tensor cores as warp-level mma
// tiles (m16n8k16, fp32 accumulate) instead of per-lane FMAs:
//   * S = K Q^T: the 16 keys are the tile's rows, D its k-steps, the group's heads (padded to 8) its
//     columns; K comes from the stage with ldmatrix (each key row's 16-byte pieces XOR-swizzled by the
//     row index as the copies land, so an ldmatrix phase hits eight bank groups), Q sits in registers;
//   * the running maximum moves only when some logit passes it by more than 8 (base 2), which one warp
//     vote decides; otherwise the chunk's probabilities 2^(l - m) (at most 2^8) are taken against the
//     maximum as it stands.  A maximum that differs from the true one cancels in O / S and M + log2 S;
//   * O^T += V^T P: D is the tile's rows (ldmatrix.trans of the V rows), the keys its k-steps and the
//     heads its columns; P goes in as a bf16 high part plus a bf16 remainder (two mma per tile), so the
//     products keep 16 bits of P's mantissa, and reaches the B-operand layout by an 8x8 register
//     transpose (movmatrix) of the S accumulator's [key][head] pairs.
// A lane then holds the heads 2 (lane % 4), + 1 of keys lane / 4 and lane / 4 + 8; the kept logits go to
// TMEM two to a lane at G' = 4 (the lanes with bit 1 set take the second key from lane ^ 2, the other lanes'
// heads being padding), all four at G' = 8, and one to each lane of a group at G' <= 2 (only the group's
// first lane holds real heads).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxGroup = 8;
constexpr int kMaxCluster = 8;
constexpr int kMaxD = 128;
constexpr int kMaxRing = 4;                 // stages per warp
constexpr int kOrderRows = 1024;            // rows up to this many are taken longest first
constexpr int kTmRing = 3;                  // stages per warp with the logits in TMEM
constexpr int kTmMinCluster = 1;            // smallest cluster of the TMEM plan
constexpr float kLn2 = 0.6931471805599453f;

struct DecodeArgs {
    CacheView c;
    const void *q;        // [S][L][Hq][D], cache dtype
    const int32_t *q_pos; // [S]
    int32_t num_q_heads, group;
    float *out;           // [S][L][Hq][D]
    float *lse;           // [S][L][Hq]
    float *scores;        // [rows][max_slots] or null
    int32_t accumulate;
    int32_t chunk;        // CH: slots per chunk (divides page_size, at most 16)
    int32_t ring;         // RW: stages per warp
    int32_t slice_cap;    // slots per CTA the logits buffer holds (multiple of CH)
    float scale_log2;     // log2(e) / sqrt(D)
    int32_t *status;
    int32_t order_rows;   // clusters take the rows longest first (rows <= kOrderRows)
};

struct DecodeShared {
    float wm[kWarps][kMaxGroup], ws[kWarps][kMaxGroup];  // per-warp running max and sum
    float pmax[kMaxGroup], psum[kMaxGroup];              // published CTA max and sum
    float pout[kMaxGroup * kMaxD];                       // published CTA output [g][d]
    float M[kMaxGroup], S[kMaxGroup];
    float pw[kWarps][16 * kMaxGroup];                    // per-warp probabilities of a chunk [key][head]
    int32_t bad;
    uint32_t tmem;                                       // TMEM base address (logits kept in TMEM)
};

// dynamic shared memory per CTA: 227 KiB per block less 9 KiB for the static part (rounded up to 128 bytes)
static_assert(sizeof(DecodeShared) + 128 <= 9 * 1024, "static shared memory");
constexpr size_t kSmemLimit = (227 - 9) * 1024;
constexpr size_t kSmemLimitTm = kSmemLimit;

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void lds8(const __nv_bfloat16 *p, float2 (&x)[4]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) x[t] = make_float2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xffff0000u));
}

__device__ __forceinline__ void lds8(const float *p, float2 (&x)[4]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    x[0] = make_float2(a.x, a.y);
    x[1] = make_float2(a.z, a.w);
    x[2] = make_float2(b.x, b.y);
    x[3] = make_float2(b.z, b.w);
}

// tensor-memory stores and loads of one warp's 32 lanes (32x32b shape: thread t owns TMEM lane base + t)
__device__ __forceinline__ void tm_st(uint32_t taddr, const float (&v)[1]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v[0])) : "memory");
}
__device__ __forceinline__ void tm_st(uint32_t taddr, const float (&v)[2]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(__float_as_uint(v[0])),
                 "r"(__float_as_uint(v[1])) : "memory");
}
__device__ __forceinline__ void tm_st(uint32_t taddr, const float (&v)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])) : "memory");
}
__device__ __forceinline__ void tm_ld8(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr) : "memory");
}
// after tcgen05.wait::ld: ties the loaded registers to a point after the wait
__device__ __forceinline__ void tm_hold8(uint32_t *r) {
    asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
}

// warp-level tensor-core steps of the bf16 path (one 16-key chunk per warp; see decode_kernel)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
// c += A (16 x 16, row) * B (16 x 8, col), bf16 operands, fp32 accumulate
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
// (x, y) -> bf16x2 with x in the low half, and the rounding remainders as a second bf16x2
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x - __low2float(h), y - __high2float(h));
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^(x - ref): zero for x = -inf (an empty max or a masked logit), whatever ref is; ref is finite otherwise
__device__ __forceinline__ float weight(float x, float ref) { return x == -INFINITY ? 0.f : ex2(x - ref); }

template <typename T, int D, int GM, int RW, bool TM, bool MM>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(DecodeArgs a) {
    constexpr int LK = D / 8;        // lanes per key
    constexpr int KW = 32 / LK;      // keys per warp step
    constexpr int MAXSTEPS = 16 / KW;
    // reduce-scatter of the dot products when every lane can end with whole ones and the partials fit
    constexpr bool kRS = MAXSTEPS * GM >= LK && MAXSTEPS * GM <= 32;
    static_assert(!TM || MM || (kRS && LK == 2 * MAXSTEPS),
                  "TMEM logits need the reduce-scatter with two lanes per key, or the tensor-core chunks");
    // MM: the chunk's two contractions on the tensor cores (bf16, groups of 4 or 8 heads, 16-slot chunks, logits
    // in TMEM)
    static_assert(!MM || (TM && sizeof(T) == 2), "tensor-core chunks: bf16, logits in TMEM");
    // TMEM logits: a lane keeps RL logits per chunk in columns [i * RL, i * RL + RL) of its warp's 256, and the
    // old score it adds in column kTmCap * RL + i: two lanes per key (reduce-scatter, RL = G' / 2; MM at G' <= 2,
    // RL = 1; MM at G' = 4, RL = 2), or (MM at G' = 8) four lanes per pair of keys, RL = 4
    constexpr int RL = MM ? (GM <= 2 ? 1 : GM / 2) : (kRS ? MAXSTEPS * GM / LK : 1);
    constexpr int kTmCap = (256 / (RL + 1)) / 8 * 8;  // chunks per warp the columns hold (a multiple of 8)
    constexpr int RB = D * (int)sizeof(T);  // bytes of a key's row
    constexpr int NS = D / 16;              // k-steps of q . k, 16-row tiles of the output
    constexpr float kSlack = 8.f;           // MM: the running maximum moves only when a logit passes it by 8 (log2)
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ DecodeShared sh;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank(), C = (int)cl.num_blocks();
    const CacheView &c = a.c;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the cluster's row: the one at its index, or (order_rows) the one whose length ranks there, longest first
    // (ties by row index), so that the longest rows start first and the launch ends evenly; every CTA of the
    // cluster ranks the same lengths and picks the same row
    int row_pick = blockIdx.x / C;
    if (a.order_rows) {
        int *lens = reinterpret_cast<int *>(smem);  // the stages are not in use yet
        __shared__ int picked;
        const int R = c.rows;
        for (int r = tid; r < R; r += kThreads) {
            const int n = c.row_len[r];
            lens[r] = (n < 0 || n > c.max_slots) ? 0 : n;
        }
        __syncthreads();
        for (int r = tid; r < R; r += kThreads) {
            const int n = lens[r];
            int above = 0;
            for (int q = 0; q < R; ++q) {
                const int m = lens[q];
                above += (m > n || (m == n && q < r)) ? 1 : 0;
            }
            if (above == row_pick) picked = r;
        }
        __syncthreads();
        row_pick = picked;
    }
    const int row = row_pick;
    const int G = a.group, Hkv = c.num_kv_heads, CH = a.chunk, P = c.page_size;
    const int seq = row / (c.num_layers * Hkv), layer = (row / Hkv) % c.num_layers, kvh = row % Hkv;
    const uint32_t half = (uint32_t)CH * D * sizeof(T);   // bytes of a chunk's K (or V)
    // a stage: the chunk's K and V rows, then (TMEM logits) its CH slot positions and CH old scores
    const uint32_t stage_bytes = TM ? 2 * half + 8 * (uint32_t)CH : 2 * half;
    unsigned char *ring = smem + (size_t)warp * RW * stage_bytes;                      // this warp's stages
    float *lg = reinterpret_cast<float *>(smem + (size_t)kWarps * RW * stage_bytes);   // [GM][slice_cap]
    int32_t *ps = reinterpret_cast<int32_t *>(lg + (size_t)GM * a.slice_cap);          // [slice_cap] positions

    int n = c.row_len[row];
    if (n < 0 || n > c.max_slots) {
        if (rank == 0 && tid == 0) report(a.status, KVC_DEV_BAD_LENGTH, row);
        n = 0;  // the row still takes part in the cluster steps, with no keys
    }
    const int nch_row = (n + CH - 1) / CH;
    const int per = (nch_row + C - 1) / C;
    const int j0 = min(nch_row, rank * per), nch = min(nch_row, j0 + per) - j0;
    const int lo = j0 * CH, cnt = min(n, (j0 + nch) * CH) - lo;
    const int qpos = a.q_pos[seq];
    const int64_t hbase = (int64_t)(seq * c.num_layers + layer) * a.num_q_heads + kvh * G;  // the group's first head
    const int32_t *bt = c.block_table + (int64_t)row * c.max_pages_per_row;
    const T *kp = static_cast<const T *>(c.k_pool);
    const T *vp = static_cast<const T *>(c.v_pool);
    const int ni = nch > warp ? (nch - warp + kWarps - 1) / kWarps : 0;  // this warp's chunks
    if (tid == 0) sh.bad = 0;
    const bool acc_old = TM && a.scores != nullptr && a.accumulate;

    // page ids of this warp's chunks, 32 at a time (one per lane): batch b sits in pb[b & 1], and batch b + 1 is
    // loaded when the first chunk of batch b is issued
    auto page_of = [&](int i) -> int { return i < ni ? bt[(lo + (warp + i * kWarps) * CH) / P] : -1; };
    int pb0 = page_of(lane), pb1 = page_of(32 + lane);
    uint32_t okmask = 0;  // bit s: stage s holds a readable page
    bool bad = false;
    auto issue = [&](int i) {
        if (i < ni) {
            const int pg = __shfl_sync(0xffffffffu, ((i >> 5) & 1) ? pb1 : pb0, i & 31);
            const int s = i % RW;
            const bool ok = pg >= 0 && pg < c.num_pages;
            okmask = ok ? (okmask | (1u << s)) : (okmask & ~(1u << s));
            const uint32_t dst = smem_u32(ring + (size_t)s * stage_bytes);
            if (ok) {
                const int64_t off = ((int64_t)pg * P + (lo + (warp + i * kWarps) * CH) % P) * D;
                const char *ks = reinterpret_cast<const char *>(kp + off);
                const char *vs = reinterpret_cast<const char *>(vp + off);
                for (uint32_t b = lane * 16; b < half; b += 512) {
                    // MM: 16-byte piece c of key row r lands at piece c ^ (r & 7), so that the eight rows an
                    // ldmatrix phase reads fall in distinct bank groups
                    const uint32_t db = MM ? (b & ~(uint32_t)(RB - 1)) |
                                                 ((((b & (RB - 1)) >> 4) ^ ((b / RB) & 7)) << 4)
                                           : b;
                    cp16(dst + db, ks + b);
                    cp16(dst + half + db, vs + b);
                }
            } else {
                bad = true;
            }
            if constexpr (TM) {
                // the chunk's slot positions and old scores, 16 bytes a lane (CH is a multiple of 4 and divides
                // max_slots, so a whole chunk lies inside the row)
                const int64_t cs = (int64_t)row * c.max_slots + lo + (warp + i * kWarps) * CH;
                const int nq = CH / 4;
                if (lane < nq) cp16(dst + 2 * half + lane * 16, c.slot_pos + cs + lane * 4);
                else if (acc_old && lane >= 16 && lane < 16 + nq)
                    cp16(dst + 2 * half + CH * 4 + (lane - 16) * 16, a.scores + cs + (lane - 16) * 4);
            }
        }
        cp_commit();  // one group per issue, empty or not, so that the group count stays in step
    };
#pragma unroll
    for (int i = 0; i < RW - 1; ++i) issue(i);

    // the slice's slot positions and the group's query slice
    const int kslot = lane / LK, sub = lane % LK;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots + lo;
    if constexpr (!TM)
        for (int i = tid; i < cnt; i += kThreads) ps[i] = pos[i];
    float2 qv[GM][4];
    {
        const T *qg = static_cast<const T *>(a.q) + hbase * D + sub * 8;
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            if (g < G) {
                float tmp[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) tmp[t] = static_cast<float>(qg[g * D + t]);
#pragma unroll
                for (int t = 0; t < 4; ++t) qv[g][t] = make_float2(tmp[2 * t], tmp[2 * t + 1]);
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t) qv[g][t] = make_float2(0.f, 0.f);
            }
        }
    }
    if constexpr (TM) {
        if (warp == 0) {  // one CTA per SM (its shared memory), so all 512 columns are free
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem)),
                         "r"(512) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    }
    __syncthreads();
    uint32_t tmw = 0;  // this warp's TMEM columns: lane quadrant warp % 4, column half warp / 4
    if constexpr (TM) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        tmw = sh.tmem + (((uint32_t)(warp & 3) * 32) << 16) + (uint32_t)(warp >> 2) * 256;
    }

    float m[GM], s[GM];
    float2 o[GM][4];
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        m[g] = -INFINITY;
        s[g] = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) o[g][t] = make_float2(0.f, 0.f);
    }
    // MM state.  A lane holds the heads hm = 2 (lane % 4), hm + 1: their running maxima and sums, and the output
    // tile entries O[d][h] for d = 16 j + lane / 4 (+ 8), h = hm, hm + 1 (the mma accumulator layout); the query
    // slice as the mma B fragments, Q[lane / 4][16 t + 2 (lane % 4) + (0, 1, 8, 9)]
    float mm[2] = {-INFINITY, -INFINITY}, ms[2] = {0.f, 0.f};
    float oc[MM ? NS : 1][4];
    uint32_t qb[MM ? NS : 1][2];
    if constexpr (MM) {
        const int hq = lane >> 2;
        const uint32_t *qg = reinterpret_cast<const uint32_t *>(static_cast<const T *>(a.q) + (hbase + hq) * D);
#pragma unroll
        for (int t = 0; t < NS; ++t) {
            qb[t][0] = hq < G ? qg[8 * t + (lane & 3)] : 0u;
            qb[t][1] = hq < G ? qg[8 * t + 4 + (lane & 3)] : 0u;
#pragma unroll
            for (int u = 0; u < 4; ++u) oc[t][u] = 0.f;
        }
    }
    const int steps = (CH + KW - 1) / KW;
    for (int i = 0; i < ni; ++i) {
        const int k = i + RW - 1;  // the chunk issued below
        if ((k & 31) == 0 && k >= 32) {
            const int b = (k >> 5) + 1;  // batch b - 1 starts here; batch b - 2, done, makes room for batch b
            if (b & 1) pb1 = page_of(b * 32 + lane);
            else pb0 = page_of(b * 32 + lane);
        }
        issue(i + RW - 1);
        cp_wait<RW - 1>();  // this lane's copies of chunk i have landed
        __syncwarp();       // and so have the other lanes'
        const int st = i % RW;
        const bool page_ok = (okmask >> st) & 1u;
        const T *Ks = reinterpret_cast<const T *>(ring + (size_t)st * stage_bytes);
        const T *Vs = Ks + CH * D;
        const int32_t *psS = reinterpret_cast<const int32_t *>(ring + (size_t)st * stage_bytes + 2 * half);
        const int il0 = (warp + i * kWarps) * CH;
        if constexpr (MM) {
            const uint32_t kb = smem_u32(Ks), vb = smem_u32(Vs);
            if (!page_ok || il0 + 16 > cnt) {  // V rows no key may use are zeroed: P is 0 there, and 0 * NaN is not
                for (int e = lane; e < 16 * RB / 16; e += 32) {
                    const int key = e / (RB / 16);
                    if (!page_ok || il0 + key >= cnt)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + e * 16), "r"(0u) : "memory");
                }
                __syncwarp();
            }
            // S[key][head] = K (16 keys x D) . Q^T: ldmatrix phase q reads keys (lane & 7) + 8 (q & 1), D piece 2t + q / 2
            float sc4[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
                const uint32_t rowa = kb + key * RB;
#pragma unroll
                for (int t = 0; t < NS; ++t) {
                    uint32_t af[4];
                    ldsm_x4(rowa + ((((uint32_t)(2 * t + (lane >> 4))) ^ (key & 7)) << 4), af);
                    mma16816(sc4, af, qb[t][0], qb[t][1]);
                }
            }
            // lane: keys ka = lane / 4 and ka + 8, heads hm, hm + 1; base-2 logits, hidden keys -inf
            const int ka = lane >> 2;
            const bool va = page_ok && il0 + ka < cnt && psS[ka] <= qpos;
            const bool vb8 = page_ok && il0 + ka + 8 < cnt && psS[ka + 8] <= qpos;
            const float l00 = va ? sc4[0] * a.scale_log2 : -INFINITY, l01 = va ? sc4[1] * a.scale_log2 : -INFINITY;
            const float l10 = vb8 ? sc4[2] * a.scale_log2 : -INFINITY, l11 = vb8 ? sc4[3] * a.scale_log2 : -INFINITY;
            float lm0 = fmaxf(l00, l10), lm1 = fmaxf(l01, l11);
            if (__any_sync(0xffffffffu, lm0 > mm[0] + kSlack || lm1 > mm[1] + kSlack)) {
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    lm0 = fmaxf(lm0, __shfl_xor_sync(0xffffffffu, lm0, off));
                    lm1 = fmaxf(lm1, __shfl_xor_sync(0xffffffffu, lm1, off));
                }
                const float n0 = fmaxf(mm[0], lm0), n1 = fmaxf(mm[1], lm1);
                const float f0 = weight(mm[0], n0), f1 = weight(mm[1], n1);
                ms[0] *= f0;
                ms[1] *= f1;
#pragma unroll
                for (int t = 0; t < NS; ++t) {
                    oc[t][0] *= f0;
                    oc[t][1] *= f1;
                    oc[t][2] *= f0;
                    oc[t][3] *= f1;
                }
                mm[0] = n0;
                mm[1] = n1;
            }
            const float p00 = weight(l00, mm[0]), p01 = weight(l01, mm[1]);
            const float p10 = weight(l10, mm[0]), p11 = weight(l11, mm[1]);
            ms[0] += p00 + p10;
            ms[1] += p01 + p11;
            if constexpr (TM) {
                if (a.scores) {
                    if constexpr (GM <= 2) {
                        // only lane 4 (lane / 4) holds real heads (0, 1): its four logits go one to each lane of
                        // its group, lane L taking value L % 4 (key ka + 8 (L % 4 / 2), head L % 2)
                        const int src = lane & ~3, v = lane & 3;
                        const float x0 = __shfl_sync(0xffffffffu, l00, src), x1 = __shfl_sync(0xffffffffu, l01, src);
                        const float x2 = __shfl_sync(0xffffffffu, l10, src), x3 = __shfl_sync(0xffffffffu, l11, src);
                        const float lv[1] = {v == 0 ? x0 : v == 1 ? x1 : v == 2 ? x2 : x3};
                        tm_st(tmw + (uint32_t)(i * RL), lv);
                        if (acc_old) {
                            const float ov[1] = {reinterpret_cast<const float *>(psS + CH)[ka + ((v & 2) ? 8 : 0)]};
                            tm_st(tmw + (uint32_t)(kTmCap * RL + i), ov);
                        }
                    } else if constexpr (GM == 4) {  // key ka (+ 8 on lanes with bit 1 set, from lane ^ 2), old score
                        const bool up = (lane & 2) != 0;
                        const float x0 = __shfl_xor_sync(0xffffffffu, l10, 2), x1 = __shfl_xor_sync(0xffffffffu, l11, 2);
                        const float lv[2] = {up ? x0 : l00, up ? x1 : l01};
                        tm_st(tmw + (uint32_t)(i * RL), lv);
                        if (acc_old) {
                            const float ov[1] = {reinterpret_cast<const float *>(psS + CH)[ka + (up ? 8 : 0)]};
                            tm_st(tmw + (uint32_t)(kTmCap * RL + i), ov);
                        }
                    } else {  // all eight heads are real: keys ka and ka + 8, heads hm, hm + 1; old score of ka (+ 8)
                        const float lv[4] = {l00, l01, l10, l11};
                        tm_st(tmw + (uint32_t)(i * RL), lv);
                        if (acc_old) {
                            const float ov[1] = {reinterpret_cast<const float *>(psS + CH)[ka + ((lane & 1) ? 8 : 0)]};
                            tm_st(tmw + (uint32_t)(kTmCap * RL + i), ov);
                        }
                    }
                }
            }
            // P as the B operand [key][head]: bf16 hi + lo (so that P keeps 16 bits of mantissa), transposed from
            // the [key][head] rows this lane holds into the [head][key] columns the fragment wants
            uint32_t h0, g0, h1, g1;
            split_bf16(p00, p01, h0, g0);
            split_bf16(p10, p11, h1, g1);
            h0 = movm_t(h0);
            g0 = movm_t(g0);
            h1 = movm_t(h1);
            g1 = movm_t(g1);
            // O^T[d][head] += V^T (d x 16 keys) . P: ldmatrix.trans phase q reads keys (lane & 7) + 8 (q / 2),
            // D piece 2t + (q & 1)
            {
                const int key = (lane & 7) + ((lane >> 4) & 1) * 8;
                const uint32_t rowa = vb + key * RB;
#pragma unroll
                for (int t = 0; t < NS; ++t) {
                    uint32_t af[4];
                    ldsm_x4_t(rowa + ((((uint32_t)(2 * t + ((lane >> 3) & 1))) ^ (key & 7)) << 4), af);
                    mma16816(oc[t], af, h0, h1);
                    mma16816(oc[t], af, g0, g1);
                }
            }
        } else if constexpr (kRS) {
            // the chunk's V = MAXSTEPS * GM partial dots per lane, reduced over the key's LK lanes by halving:
            // lane sub ends with the R complete dots v = sub * R + r (step v / GM, head v % GM)
            constexpr int V = MAXSTEPS * GM, R = V / LK;
            float d[V];
            uint32_t vis = 0;
#pragma unroll
            for (int t = 0; t < MAXSTEPS; ++t) {
                const int kk = t * KW + kslot;
                const bool v = t < steps && page_ok && kk < CH && il0 + kk < cnt &&
                               (TM ? psS[kk] : ps[il0 + kk]) <= qpos;
                vis |= (v ? 1u : 0u) << t;
                float2 x[4];
                if (v) lds8(Ks + kk * D + sub * 8, x);
                else
#pragma unroll
                    for (int u = 0; u < 4; ++u) x[u] = make_float2(0.f, 0.f);
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    float2 acc = __fmul2_rn(qv[g][0], x[0]);
                    acc = __ffma2_rn(qv[g][1], x[1], acc);
                    acc = __ffma2_rn(qv[g][2], x[2], acc);
                    acc = __ffma2_rn(qv[g][3], x[3], acc);
                    d[t * GM + g] = acc.x + acc.y;
                }
            }
#pragma unroll
            for (int lvl = 0; (LK >> (lvl + 1)) > 0; ++lvl) {
                const int off = LK >> (lvl + 1), n = V >> (lvl + 1);
                const bool up = (sub & off) != 0;
#pragma unroll
                for (int r = 0; r < n; ++r) {
                    const float keep = up ? d[r + n] : d[r];
                    const float send = up ? d[r] : d[r + n];
                    d[r] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            const int vbase = sub * R;
            float lv[R];
            float cm[GM];
#pragma unroll
            for (int g = 0; g < GM; ++g) cm[g] = -INFINITY;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int v = vbase + r, t = v / GM, g = v % GM, kk = t * KW + kslot;
                lv[r] = ((vis >> t) & 1u) ? d[r] * a.scale_log2 : -INFINITY;
                if (!TM && g < G && t < steps && kk < CH && il0 + kk < cnt) lg[(size_t)g * a.slice_cap + il0 + kk] = lv[r];
#pragma unroll
                for (int h = 0; h < GM; ++h)
                    if (h == g) cm[h] = fmaxf(cm[h], lv[r]);
            }
            if constexpr (TM) {
                if (a.scores) {  // the lane's logits of chunk i, and the old score of the key its lane pair sums
                    tm_st(tmw + (uint32_t)(i * R), lv);
                    if (acc_old) {
                        const int ko = (sub >> 1) * KW + kslot;
                        const float ov[1] = {ko < CH ? reinterpret_cast<const float *>(psS + CH)[ko] : 0.f};
                        tm_st(tmw + (uint32_t)(kTmCap * R + i), ov);
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                cm[g] = warp_max(cm[g]);
                const float mn = fmaxf(m[g], cm[g]);
                if (mn != m[g]) {  // warp-uniform: a new maximum rescales the running sums and output
                    const float f = weight(m[g], mn);
                    s[g] *= f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) o[g][u] = __fmul2_rn(o[g][u], make_float2(f, f));
                    m[g] = mn;
                }
            }
            // one exponential per (key, head); the key's lanes read all its heads' probabilities back
            float *pwv = sh.pw[warp];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int v = vbase + r, t = v / GM, g = v % GM;
                float mg = m[0];
#pragma unroll
                for (int h = 1; h < GM; ++h)
                    if (h == g) mg = m[h];
                const float p = lv[r] == -INFINITY ? 0.f : ex2(lv[r] - mg);
#pragma unroll
                for (int h = 0; h < GM; ++h)
                    if (h == g) s[h] += p;
                pwv[(t * KW + kslot) * GM + g] = p;
            }
            __syncwarp();
#pragma unroll
            for (int t = 0; t < MAXSTEPS; ++t) {
                if ((vis >> t) & 1u) {
                    const int kk = t * KW + kslot;
                    float2 y[4];
                    lds8(Vs + kk * D + sub * 8, y);
                    float pp[GM];
                    const float *src = pwv + kk * GM;
                    if constexpr (GM % 4 == 0) {
#pragma unroll
                        for (int h = 0; h < GM; h += 4) {
                            const float4 f4 = *reinterpret_cast<const float4 *>(src + h);
                            pp[h] = f4.x; pp[h + 1] = f4.y; pp[h + 2] = f4.z; pp[h + 3] = f4.w;
                        }
                    } else {
#pragma unroll
                        for (int h = 0; h < GM; ++h) pp[h] = src[h];
                    }
#pragma unroll
                    for (int g = 0; g < GM; ++g)
#pragma unroll
                        for (int u = 0; u < 4; ++u) o[g][u] = __ffma2_rn(make_float2(pp[g], pp[g]), y[u], o[g][u]);
                }
            }
        } else {
            float l[MAXSTEPS][GM];
            uint32_t vis = 0;
            float cm[GM];
    #pragma unroll
            for (int g = 0; g < GM; ++g) cm[g] = -INFINITY;
    #pragma unroll
            for (int t = 0; t < MAXSTEPS; ++t) {
                if (t < steps) {
                    const int kk = t * KW + kslot;
                    const bool in = kk < CH && il0 + kk < cnt;
                    const bool v = page_ok && in && ps[il0 + kk] <= qpos;
                    vis |= (v ? 1u : 0u) << t;
                    float2 x[4];
                    if (v) lds8(Ks + kk * D + sub * 8, x);
                    else
    #pragma unroll
                        for (int u = 0; u < 4; ++u) x[u] = make_float2(0.f, 0.f);
    #pragma unroll
                    for (int g = 0; g < GM; ++g) {
                        float2 acc = __fmul2_rn(qv[g][0], x[0]);
                        acc = __ffma2_rn(qv[g][1], x[1], acc);
                        acc = __ffma2_rn(qv[g][2], x[2], acc);
                        acc = __ffma2_rn(qv[g][3], x[3], acc);
                        float d = acc.x + acc.y;
    #pragma unroll
                        for (int off = LK / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                        const float lv = v ? d * a.scale_log2 : -INFINITY;
                        l[t][g] = lv;
                        if (g < G && in && sub == 0) lg[(size_t)g * a.slice_cap + il0 + kk] = lv;
                        cm[g] = fmaxf(cm[g], lv);
                    }
                }
            }
    #pragma unroll
            for (int g = 0; g < GM; ++g) {
    #pragma unroll
                for (int off = LK; off < 32; off <<= 1) cm[g] = fmaxf(cm[g], __shfl_xor_sync(0xffffffffu, cm[g], off));
                const float mn = fmaxf(m[g], cm[g]);
                if (mn != m[g]) {  // warp-uniform: a new maximum rescales the running sum and output
                    const float f = weight(m[g], mn);
                    s[g] *= f;
    #pragma unroll
                    for (int u = 0; u < 4; ++u) o[g][u] = __fmul2_rn(o[g][u], make_float2(f, f));
                    m[g] = mn;
                }
            }
    #pragma unroll
            for (int t = 0; t < MAXSTEPS; ++t) {
                if (t < steps && ((vis >> t) & 1u)) {
                    const int kk = t * KW + kslot;
                    float2 y[4];
                    lds8(Vs + kk * D + sub * 8, y);
    #pragma unroll
                    for (int g = 0; g < GM; ++g) {
                        const float p = ex2(l[t][g] - m[g]);
                        s[g] += p;
    #pragma unroll
                        for (int u = 0; u < 4; ++u) o[g][u] = __ffma2_rn(make_float2(p, p), y[u], o[g][u]);
                    }
                }
            }
        }
        __syncwarp();  // every lane is done with stage st before the next issue refills it
    }
    cp_wait<0>();
    if constexpr (MM) {  // the sums over the lanes that share heads; the maxima already agree across them
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            ms[0] += __shfl_xor_sync(0xffffffffu, ms[0], off);
            ms[1] += __shfl_xor_sync(0xffffffffu, ms[1], off);
        }
        if (lane < (GM + 1) / 2) {
            sh.wm[warp][2 * lane] = mm[0];
            sh.wm[warp][2 * lane + 1] = mm[1];
            sh.ws[warp][2 * lane] = ms[0];
            sh.ws[warp][2 * lane + 1] = ms[1];
        }
        if (lane == 0 && bad) sh.bad = 1;
    }
    // the warp's totals: the output over its key lanes (lanes that share sub); the sum over the lanes that
    // hold distinct probabilities (all of them after the reduce-scatter, else one lane group per key)
#pragma unroll
    for (int g = 0; g < (MM ? 0 : GM); ++g) {
        if constexpr (kRS) {
#pragma unroll
            for (int off = 1; off < LK; off <<= 1) s[g] += __shfl_xor_sync(0xffffffffu, s[g], off);
        }
#pragma unroll
        for (int off = LK; off < 32; off <<= 1) {
            s[g] += __shfl_xor_sync(0xffffffffu, s[g], off);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                o[g][u].x += __shfl_xor_sync(0xffffffffu, o[g][u].x, off);
                o[g][u].y += __shfl_xor_sync(0xffffffffu, o[g][u].y, off);
            }
        }
    }
    if (!MM && lane == 0) {
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            sh.wm[warp][g] = m[g];
            sh.ws[warp][g] = s[g];
        }
        if (bad) sh.bad = 1;
    }
    __syncthreads();  // every warp is past its last chunk: the stages take the partial outputs
    float *wo = reinterpret_cast<float *>(smem);  // [kWarps][G][D]
    if constexpr (MM) {
        const int hm = 2 * (lane & 3);
#pragma unroll
        for (int t = 0; t < NS; ++t) {
            const int d = 16 * t + (lane >> 2);
            if (hm < G) {
                wo[((size_t)warp * G + hm) * D + d] = oc[t][0];
                wo[((size_t)warp * G + hm) * D + d + 8] = oc[t][2];
            }
            if (hm + 1 < G) {
                wo[((size_t)warp * G + hm + 1) * D + d] = oc[t][1];
                wo[((size_t)warp * G + hm + 1) * D + d + 8] = oc[t][3];
            }
        }
    }
    if (!MM && kslot == 0)
#pragma unroll
        for (int g = 0; g < GM; ++g)
            if (g < G)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    wo[((size_t)warp * G + g) * D + sub * 8 + 2 * u] = o[g][u].x;
                    wo[((size_t)warp * G + g) * D + sub * 8 + 2 * u + 1] = o[g][u].y;
                }
    if (tid < GM) {
        float mx = -INFINITY;
        for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, sh.wm[w][tid]);
        float sm = 0.f;
        for (int w = 0; w < kWarps; ++w) sm += sh.ws[w][tid] * weight(sh.wm[w][tid], mx);
        sh.pmax[tid] = mx;
        sh.psum[tid] = sm;
    }
    __syncthreads();
    // CTA totals in warp order
    for (int e = tid; e < G * D; e += kThreads) {
        const int g = e / D;
        float acc = 0.f;
        for (int w = 0; w < kWarps; ++w) acc += wo[(size_t)w * G * D + e] * weight(sh.wm[w][g], sh.pmax[g]);
        sh.pout[e] = acc;
    }
    cl.sync();

    // cluster totals in rank order
    if (tid < GM) {
        float mx = -INFINITY;
        for (int r = 0; r < C; ++r) mx = fmaxf(mx, cl.map_shared_rank(&sh, r)->pmax[tid]);
        float sm = 0.f;
        for (int r = 0; r < C; ++r) {
            const DecodeShared *o = cl.map_shared_rank(&sh, r);
            sm += o->psum[tid] * weight(o->pmax[tid], mx);
        }
        sh.M[tid] = mx;
        sh.S[tid] = sm;
    }
    __syncthreads();
    if (rank == 0) {
        for (int e = tid; e < G * D; e += kThreads) {
            const int g = e / D;
            float acc = 0.f;
            for (int r = 0; r < C; ++r) {
                const DecodeShared *o = cl.map_shared_rank(&sh, r);
                acc += o->pout[e] * weight(o->pmax[g], sh.M[g]);
            }
            a.out[hbase * D + e] = sh.S[g] > 0.f ? acc / sh.S[g] : 0.f;
        }
        if (tid < G) a.lse[hbase + tid] = sh.S[tid] > 0.f ? (sh.M[tid] + log2f(sh.S[tid])) * kLn2 : -INFINITY;
        if (tid == 0) {
            bool bad = false;
            for (int r = 0; r < C; ++r) bad |= cl.map_shared_rank(&sh, r)->bad != 0;
            if (bad) report(a.status, KVC_DEV_BAD_PAGE, row);
        }
    }
    if (MM && GM <= 2 && a.scores) {
        // lane L holds key L / 4 + 8 (L % 4 / 2), head L % 2: the pair L, L ^ 1 sums the key's heads
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        const int hh = lane & 1;
        const float inv = (hh < G && sh.S[hh] > 0.f) ? 1.f / sh.S[hh] : 0.f, mg = sh.M[hh];
        const int ko = (lane >> 2) + ((lane & 2) ? 8 : 0);
        float *sc = a.scores + (int64_t)row * c.max_slots + lo;
        for (int i0 = 0; i0 < ni; i0 += 8) {
            uint32_t lr[8], orr[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            tm_ld8(tmw + (uint32_t)(i0 * RL), lr);
            if (acc_old) tm_ld8(tmw + (uint32_t)(kTmCap * RL + i0), orr);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            tm_hold8(lr);
            tm_hold8(orr);
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                float part = hh < G ? weight(__uint_as_float(lr[b]), mg) * inv : 0.f;
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                const int il = (warp + (i0 + b) * kWarps) * CH + ko;
                if (i0 + b < ni && hh == 0 && il < cnt) sc[il] = __uint_as_float(orr[b]) + part;
            }
        }
    }
    if (MM && GM == 8 && a.scores) {
        // lane L holds keys L / 4 and L / 4 + 8, heads 2 (L % 4), + 1: the four lanes of L / 4 sum both keys'
        // heads; lane 4 (L / 4) writes the first key, lane 4 (L / 4) + 1 the second (the one whose old score it kept)
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        const int hm = 2 * (lane & 3);
        float inv[2], mg[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            inv[r] = (hm + r < G && sh.S[hm + r] > 0.f) ? 1.f / sh.S[hm + r] : 0.f;
            mg[r] = sh.M[hm + r];
        }
        const int ko = (lane >> 2) + ((lane & 1) ? 8 : 0);
        float *sc = a.scores + (int64_t)row * c.max_slots + lo;
        for (int i0 = 0; i0 < ni; i0 += 8) {
            uint32_t lr[32], orr[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
            for (int b = 0; b < 4; ++b) tm_ld8(tmw + (uint32_t)(i0 * RL + 8 * b), lr + 8 * b);
            if (acc_old) tm_ld8(tmw + (uint32_t)(kTmCap * RL + i0), orr);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int b = 0; b < 4; ++b) tm_hold8(lr + 8 * b);
            tm_hold8(orr);
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                float pa = 0.f, pb = 0.f;
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    if (hm + r < G) {
                        pa = fmaf(weight(__uint_as_float(lr[4 * b + r]), mg[r]), inv[r], pa);
                        pb = fmaf(weight(__uint_as_float(lr[4 * b + 2 + r]), mg[r]), inv[r], pb);
                    }
                pa += __shfl_xor_sync(0xffffffffu, pa, 1);
                pb += __shfl_xor_sync(0xffffffffu, pb, 1);
                pa += __shfl_xor_sync(0xffffffffu, pa, 2);
                pb += __shfl_xor_sync(0xffffffffu, pb, 2);
                const int il = (warp + (i0 + b) * kWarps) * CH + ko;
                if (i0 + b < ni && (lane & 3) < 2 && il < cnt)
                    sc[il] = __uint_as_float(orr[b]) + ((lane & 1) ? pb : pa);
            }
        }
    }
    if (MM && GM == 4 && a.scores) {
        // lane L holds key (L / 4) + 8 ((L >> 1) & 1), heads 2 (L & 1), + 1: the pair L, L ^ 1 sums the key's heads
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        const int hl = 2 * (lane & 1);
        float inv[2], mg[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            inv[r] = (hl + r < G && sh.S[hl + r] > 0.f) ? 1.f / sh.S[hl + r] : 0.f;
            mg[r] = sh.M[hl + r];
        }
        const int ko = (lane >> 2) + ((lane >> 1) & 1) * 8;
        float *sc = a.scores + (int64_t)row * c.max_slots + lo;
        for (int i0 = 0; i0 < ni; i0 += 8) {
            uint32_t lr[16], orr[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            tm_ld8(tmw + (uint32_t)(i0 * RL), lr);
            tm_ld8(tmw + (uint32_t)(i0 * RL + 8), lr + 8);
            if (acc_old) tm_ld8(tmw + (uint32_t)(kTmCap * RL + i0), orr);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            tm_hold8(lr);
            tm_hold8(lr + 8);
            tm_hold8(orr);
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                float part = 0.f;
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    if (hl + r < G) part = fmaf(weight(__uint_as_float(lr[2 * b + r]), mg[r]), inv[r], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                const int il = (warp + (i0 + b) * kWarps) * CH + ko;
                if (i0 + b < ni && (lane & 1) == 0 && il < cnt) sc[il] = __uint_as_float(orr[b]) + part;
            }
        }
    }
    if (TM && !MM && a.scores) {
        // each lane pair adds its key's sum over the heads, from the logits and old scores kept in TMEM
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        float inv[RL], mg[RL];
        bool use[RL];
#pragma unroll
        for (int r = 0; r < RL; ++r) {
            const int g = (sub & 1) * RL + r;  // the head of this lane's r-th logit of a key
            use[r] = g < G;
            inv[r] = (g < G && sh.S[g] > 0.f) ? 1.f / sh.S[g] : 0.f;
            mg[r] = sh.M[g];
        }
        const int ko = (sub >> 1) * KW + kslot;  // the key within a chunk
        float *sc = a.scores + (int64_t)row * c.max_slots + lo;
        for (int i0 = 0; i0 < ni; i0 += 8) {  // eight chunks a batch (kTmCap is a multiple of 8)
            uint32_t lr[8 * RL], orr[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
            for (int b = 0; b < RL; ++b) tm_ld8(tmw + (uint32_t)(i0 * RL + 8 * b), lr + 8 * b);
            if (acc_old) tm_ld8(tmw + (uint32_t)(kTmCap * RL + i0), orr);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int b = 0; b < RL; ++b) tm_hold8(lr + 8 * b);
            tm_hold8(orr);
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                float part = 0.f;
#pragma unroll
                for (int r = 0; r < RL; ++r)
                    if (use[r]) part = fmaf(weight(__uint_as_float(lr[b * RL + r]), mg[r]), inv[r], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                const int il = (warp + (i0 + b) * kWarps) * CH + ko;
                if (i0 + b < ni && (sub & 1) == 0 && ko < CH && il < cnt) sc[il] = __uint_as_float(orr[b]) + part;
            }
        }
    }
    if (!TM && a.scores) {
        float inv[GM], mg[GM];
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            inv[g] = (g < G && sh.S[g] > 0.f) ? 1.f / sh.S[g] : 0.f;
            mg[g] = sh.M[g];
        }
        float *sc = a.scores + (int64_t)row * c.max_slots + lo;
        constexpr int kBatch = 8;  // the read-modify-write loads of a batch are all in flight together
        for (int i0 = 0; i0 < cnt; i0 += kBatch * kThreads) {
            float old[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int i = i0 + b * kThreads + tid;
                old[b] = (a.accumulate && i < cnt) ? sc[i] : 0.f;
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int i = i0 + b * kThreads + tid;
                if (i >= cnt) break;
                float v = old[b];
#pragma unroll
                for (int g = 0; g < GM; ++g)
                    if (g < G) v = fmaf(weight(lg[(size_t)g * a.slice_cap + i], mg[g]), inv[g], v);
                sc[i] = v;
            }
        }
    }
    if constexpr (TM) asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cl.sync();  // peers may still be reading this CTA's shared memory
    if constexpr (TM) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sh.tmem), "r"(512) : "memory");
    }
}

int group_bound(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

struct Plan {
    int C, CH, RW, cap;
    size_t smem;
    bool tm;  // logits, slot positions and old scores through the stages and TMEM
    bool mm;  // and the chunk's contractions on the tensor cores (bf16, G' = 4, 16-slot chunks)
};

// the reduce-scatter with two lanes per key (the TMEM layout) for head size D and group bound GM
constexpr bool two_lanes_per_key(int D, int GM) {
    const int LK = D / 8, KW = 32 / LK, MAXSTEPS = 16 / KW, V = MAXSTEPS * GM;
    return V >= LK && V <= 32 && LK == 2 * MAXSTEPS;
}

// Cluster size, chunk, stages per warp and shared memory of a launch; C = 0 when nothing fits.  The chunk is
// the largest divisor of the page size, at most 16 slots, whose two stages per warp fit; the cluster grows
// (shrinking each CTA's logits buffer) until every warp has kMaxRing stages or C is 8.  At least two stages
// per warp are needed: one landing while the other is worked on.
//
// With `aligned` (slot positions and scores 16-byte aligned) and the two-lanes-per-key reduce-scatter, the
// TMEM plan comes first: three stages per warp, the smallest cluster whose warps' chunks fit the TMEM columns.
// With bf16, 16-slot chunks and a 4-byte aligned query (`q4`), the chunks' contractions run as mma tiles (their
// TMEM layout needs no reduce-scatter).
Plan plan_for(const CacheView &c, int G, int sms, bool aligned, bool q4) {
    const size_t elem = c.dtype == KVC_BF16 ? 2 : 4;
    const size_t partial = (size_t)kWarps * G * c.head_dim * 4;
    const int GM = group_bound(G);
    int C0 = 1;
    while (C0 < kMaxCluster && (int64_t)c.rows * C0 < sms) C0 <<= 1;
    const bool two = two_lanes_per_key(c.head_dim, GM);
    const bool mm_ok = q4 && c.dtype == KVC_BF16;  // tensor-core chunks (16-slot ones)
    if (aligned && (two || mm_ok)) {
        const int RL = GM <= 2 ? 1 : GM / 2, cap_w = (256 / (RL + 1)) / 8 * 8;  // the kernel's RL and kTmCap
        for (int CH = std::min(16, c.page_size); CH >= 4; --CH) {
            if (c.page_size % CH || CH % 4 || c.max_slots % CH) continue;
            const bool mm = mm_ok && CH == 16;
            if (!mm && !two) continue;
            const size_t stage = 2 * (size_t)CH * c.head_dim * elem + 8 * (size_t)CH;
            const size_t smem = (size_t)kTmRing * kWarps * stage;
            if (smem > kSmemLimitTm || smem < partial) continue;
            const int64_t nch = (c.max_slots + CH - 1) / CH;
            for (int C = std::max(C0, kTmMinCluster); C <= kMaxCluster; C <<= 1)
                if (((nch + C - 1) / C + kWarps - 1) / kWarps <= cap_w)
                    return Plan{C, CH, kTmRing, 0, smem, true, mm};
        }
    }
    for (int CH = std::min(16, c.page_size); CH >= 1; --CH) {
        if (c.page_size % CH) continue;
        const size_t stage = 2 * (size_t)CH * c.head_dim * elem;
        const int64_t nch = (c.max_slots + CH - 1) / CH;
        Plan best{};
        for (int C = C0; C <= kMaxCluster; C <<= 1) {
            const int64_t cap = ((nch + C - 1) / C) * CH;
            const size_t fixed = (size_t)(GM + 1) * cap * 4;  // logits and slot positions
            if (fixed >= kSmemLimit) continue;
            const int RW = (int)std::min<size_t>(kMaxRing, (kSmemLimit - fixed) / (kWarps * stage));
            if (RW < 2 || (size_t)RW * kWarps * stage < partial) continue;
            if (RW > best.RW) best = Plan{C, CH, RW, (int)cap, (size_t)RW * kWarps * stage + fixed, false, false};
            if (RW >= kMaxRing) break;
        }
        if (best.C) return best;
    }
    return Plan{};
}

int sm_count() { return device_sms(); }

template <typename T, int D, int GM, int RW, bool TM, bool MM>
cudaError_t launch_t(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, const Plan &p) {
    const int G = num_q_heads / c.num_kv_heads;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)decode_kernel<T, D, GM, RW, TM, MM>, p.smem, smem_set);
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    const int order = c.rows <= kOrderRows && (int64_t)c.rows * p.C > sms ? 1 : 0;  // more than one wave
    DecodeArgs a{c, q, q_pos, num_q_heads, G, out, lse, scores, accumulate ? 1 : 0, p.CH, p.RW, p.cap,
                 (float)(1.4426950408889634 / std::sqrt((double)D)), status, order};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c.rows * p.C));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<T, D, GM, RW, TM, MM>, a);
}

template <typename T, int D, int GM>
cudaError_t launch_r(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, const Plan &p) {
    if constexpr (sizeof(T) == 2) {
        if (p.mm)
            return launch_t<T, D, GM, kTmRing, true, true>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate,
                                                           status, stream, p);
    }
    if constexpr (two_lanes_per_key(D, GM)) {
        if (p.tm && !p.mm)
            return launch_t<T, D, GM, kTmRing, true, false>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate,
                                                            status, stream, p);
    }
    if (p.tm) return cudaErrorInvalidValue;
    switch (p.RW) {
        case 2: return launch_t<T, D, GM, 2, false, false>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        case 3: return launch_t<T, D, GM, 3, false, false>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        default: return launch_t<T, D, GM, 4, false, false>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
    }
}

template <typename T, int D>
cudaError_t launch_g(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, const Plan &p) {
    switch (group_bound(num_q_heads / c.num_kv_heads)) {
        case 1: return launch_r<T, D, 1>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        case 2: return launch_r<T, D, 2>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        case 4: return launch_r<T, D, 4>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        default: return launch_r<T, D, 8>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
    }
}

}  // namespace

int decode_cluster(const CacheView &c, int32_t group) {
    if (group < 1 || group > kMaxGroup) return 0;
    return plan_for(c, group, sm_count(), false, false).C;
}

cudaError_t launch_decode(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                          float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, int) {
    const bool aligned = (reinterpret_cast<uintptr_t>(c.slot_pos) & 15) == 0 &&
                         (reinterpret_cast<uintptr_t>(scores) & 15) == 0;  // a null scores pointer is aligned
    const Plan p = plan_for(c, num_q_heads / c.num_kv_heads, sm_count(), aligned,
                            (reinterpret_cast<uintptr_t>(q) & 3) == 0);
    if (p.C == 0) return cudaErrorInvalidValue;
    const bool bf16 = c.dtype == KVC_BF16;
    if (c.head_dim == 64)
        return bf16 ? launch_g<__nv_bfloat16, 64>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p)
                    : launch_g<float, 64>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
    return bf16 ? launch_g<__nv_bfloat16, 128>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p)
                : launch_g<float, 128>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
}

}  // namespace kvc
