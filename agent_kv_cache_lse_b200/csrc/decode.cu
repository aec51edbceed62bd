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
constexpr size_t kSmemLimit = 220 * 1024;   // dynamic bytes per CTA
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
};

struct DecodeShared {
    float wm[kWarps][kMaxGroup], ws[kWarps][kMaxGroup];  // per-warp running max and sum
    float pmax[kMaxGroup], psum[kMaxGroup];              // published CTA max and sum
    float pout[kMaxGroup * kMaxD];                       // published CTA output [g][d]
    float M[kMaxGroup], S[kMaxGroup];
    float pw[kWarps][16 * kMaxGroup];                    // per-warp probabilities of a chunk [key][head]
    int32_t bad;
};

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

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^(x - ref): zero for x = -inf (an empty max or a masked logit), whatever ref is; ref is finite otherwise
__device__ __forceinline__ float weight(float x, float ref) { return x == -INFINITY ? 0.f : ex2(x - ref); }

template <typename T, int D, int GM, int RW>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(DecodeArgs a) {
    constexpr int LK = D / 8;        // lanes per key
    constexpr int KW = 32 / LK;      // keys per warp step
    constexpr int MAXSTEPS = 16 / KW;
    // reduce-scatter of the dot products when every lane can end with whole ones and the partials fit
    constexpr bool kRS = MAXSTEPS * GM >= LK && MAXSTEPS * GM <= 32;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ DecodeShared sh;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank(), C = (int)cl.num_blocks();
    const int row = blockIdx.x / C;
    const CacheView &c = a.c;
    const int G = a.group, Hkv = c.num_kv_heads, CH = a.chunk, P = c.page_size;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seq = row / (c.num_layers * Hkv), layer = (row / Hkv) % c.num_layers, kvh = row % Hkv;
    const uint32_t half = (uint32_t)CH * D * sizeof(T);   // bytes of a chunk's K (or V)
    const uint32_t stage_bytes = 2 * half;
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
            if (ok) {
                const int64_t off = ((int64_t)pg * P + (lo + (warp + i * kWarps) * CH) % P) * D;
                const char *ks = reinterpret_cast<const char *>(kp + off);
                const char *vs = reinterpret_cast<const char *>(vp + off);
                const uint32_t dst = smem_u32(ring + (size_t)s * stage_bytes);
                for (uint32_t b = lane * 16; b < half; b += 512) {
                    cp16(dst + b, ks + b);
                    cp16(dst + half + b, vs + b);
                }
            } else {
                bad = true;
            }
        }
        cp_commit();  // one group per issue, empty or not, so that the group count stays in step
    };
#pragma unroll
    for (int i = 0; i < RW - 1; ++i) issue(i);

    // the slice's slot positions and the group's query slice
    const int kslot = lane / LK, sub = lane % LK;
    const int32_t *pos = c.slot_pos + (int64_t)row * c.max_slots + lo;
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
    __syncthreads();

    float m[GM], s[GM];
    float2 o[GM][4];
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        m[g] = -INFINITY;
        s[g] = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) o[g][t] = make_float2(0.f, 0.f);
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
        const int il0 = (warp + i * kWarps) * CH;
        if constexpr (kRS) {
            // the chunk's V = MAXSTEPS * GM partial dots per lane, reduced over the key's LK lanes by halving:
            // lane sub ends with the R complete dots v = sub * R + r (step v / GM, head v % GM)
            constexpr int V = MAXSTEPS * GM, R = V / LK;
            float d[V];
            uint32_t vis = 0;
#pragma unroll
            for (int t = 0; t < MAXSTEPS; ++t) {
                const int kk = t * KW + kslot;
                const bool v = t < steps && page_ok && kk < CH && il0 + kk < cnt && ps[il0 + kk] <= qpos;
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
                if (g < G && t < steps && kk < CH && il0 + kk < cnt) lg[(size_t)g * a.slice_cap + il0 + kk] = lv[r];
#pragma unroll
                for (int h = 0; h < GM; ++h)
                    if (h == g) cm[h] = fmaxf(cm[h], lv[r]);
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
    // the warp's totals: the output over its key lanes (lanes that share sub); the sum over the lanes that
    // hold distinct probabilities (all of them after the reduce-scatter, else one lane group per key)
#pragma unroll
    for (int g = 0; g < GM; ++g) {
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
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            sh.wm[warp][g] = m[g];
            sh.ws[warp][g] = s[g];
        }
        if (bad) sh.bad = 1;
    }
    __syncthreads();  // every warp is past its last chunk: the stages take the partial outputs
    float *wo = reinterpret_cast<float *>(smem);  // [kWarps][G][D]
    if (kslot == 0)
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
    if (a.scores) {
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
    cl.sync();  // peers may still be reading this CTA's shared memory
}

int group_bound(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

struct Plan {
    int C, CH, RW, cap;
    size_t smem;
};

// Cluster size, chunk, stages per warp and shared memory of a launch; C = 0 when nothing fits.  The chunk is
// the largest divisor of the page size, at most 16 slots, whose two stages per warp fit; the cluster grows
// (shrinking each CTA's logits buffer) until every warp has kMaxRing stages or C is 8.  At least two stages
// per warp are needed: one landing while the other is worked on.
Plan plan_for(const CacheView &c, int G, int sms) {
    const size_t elem = c.dtype == KVC_BF16 ? 2 : 4;
    const size_t partial = (size_t)kWarps * G * c.head_dim * 4;
    const int GM = group_bound(G);
    int C0 = 1;
    while (C0 < kMaxCluster && (int64_t)c.rows * C0 < sms) C0 <<= 1;
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
            if (RW > best.RW) best = Plan{C, CH, RW, (int)cap, (size_t)RW * kWarps * stage + fixed};
            if (RW >= kMaxRing) break;
        }
        if (best.C) return best;
    }
    return Plan{};
}

int sm_count() { return device_sms(); }

template <typename T, int D, int GM, int RW>
cudaError_t launch_t(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, const Plan &p) {
    const int G = num_q_heads / c.num_kv_heads;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)decode_kernel<T, D, GM, RW>, p.smem, smem_set);
    if (e != cudaSuccess) return e;
    DecodeArgs a{c, q, q_pos, num_q_heads, G, out, lse, scores, accumulate ? 1 : 0, p.CH, p.RW, p.cap,
                 (float)(1.4426950408889634 / std::sqrt((double)D)), status};
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
    return cudaLaunchKernelEx(&cfg, decode_kernel<T, D, GM, RW>, a);
}

template <typename T, int D, int GM>
cudaError_t launch_r(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                     float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, const Plan &p) {
    switch (p.RW) {
        case 2: return launch_t<T, D, GM, 2>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        case 3: return launch_t<T, D, GM, 3>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
        default: return launch_t<T, D, GM, 4>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
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
    return plan_for(c, group, sm_count()).C;
}

cudaError_t launch_decode(const CacheView &c, const void *q, const int32_t *q_pos, int32_t num_q_heads, float *out,
                          float *lse, float *scores, bool accumulate, int32_t *status, cudaStream_t stream, int) {
    const Plan p = plan_for(c, num_q_heads / c.num_kv_heads, sm_count());
    if (p.C == 0) return cudaErrorInvalidValue;
    const bool bf16 = c.dtype == KVC_BF16;
    if (c.head_dim == 64)
        return bf16 ? launch_g<__nv_bfloat16, 64>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p)
                    : launch_g<float, 64>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
    return bf16 ? launch_g<__nv_bfloat16, 128>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p)
                : launch_g<float, 128>(c, q, q_pos, num_q_heads, out, lse, scores, accumulate, status, stream, p);
}

}  // namespace kvc
