// Beacon-query maintenance: online k-means over each group's past queries.
//
// "BeaconKV Compresses KV Cache for Long-Reasoning Models with Beacon Queries", Key ideas:
// queries that revisit distant context fall into a few similarity groups, and one
// representative per group (a beacon query) joins the recent queries in the query set.
// The groups are kept here by online (mini-batch) k-means, separately for every
// (sequence, layer, query head); each call folds in that group's new queries:
//   1. beacons with count 0 are seeded, in index order, with the first new queries;
//   2. each new query joins its nearest beacon among those with a count or a seed;
//   3. each beacon that drew queries becomes the mean of all it has absorbed.
// The assignment is an integer decided by floating point, so it is computed in one fixed
// fp32 order that a reference can repeat exactly: distance = sum over d = 0..D-1, in
// order, of (q_d - c_d)^2 with the difference, the square and each partial sum rounded
// separately (no fused multiply-add); the lower beacon index wins a tie.  The mean is
// fp32 in a fixed order as well: S = c * n, S += each new query of the beacon in query
// order, c = S / (n + drawn).
//
// One CTA per group.  The beacons and (when they fit) the group's new queries sit in
// shared memory; each thread runs four (query, beacon) distance sums side by side; warp
// ballots list every beacon's queries in ascending order; the update runs one thread per
// (beacon, dimension) over its beacon's list.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace kvc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxBeacons = 64;
constexpr int kPairs = 4 * kThreads;  // (query, beacon) distances per round: four per thread
constexpr int kListMax = 8192;         // per-beacon query lists are built when a group brings at most this many
constexpr size_t kSmemCap = 227 * 1024;

struct BeaconArgs {
    const void *q;
    const int32_t *num_q;
    int32_t num_layers, num_q_heads, head_dim, max_q, bf16;
    float *beacons;
    int32_t *counts;
    int32_t num_beacons;
    void *beacon_q;
    int32_t out_max_q;
    int32_t stage_rows;  // rows of the query staging area (all of a group's queries when they fit)
    int32_t *status;
};

__device__ __forceinline__ float load_q(const BeaconArgs &a, int64_t idx) {
    return a.bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.q)[idx]) : static_cast<const float *>(a.q)[idx];
}

__global__ void __launch_bounds__(kThreads) beacon_kernel(BeaconArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int B = a.num_beacons, D = a.head_dim, Hq = a.num_q_heads;
    const int R = min(64, kPairs / B);                                   // queries per round of distances
    // padded rows: rows fall in different banks; with D % 4 == 0 the rows stay 16-byte aligned (4 floats of
    // padding) so that the distance sums read four dimensions per load
    const bool vec = (D & 3) == 0;
    const int DP = vec ? D + 4 : D + 1;
    float *cb = reinterpret_cast<float *>(smem_raw);                   // [B][DP] beacons
    float *qs = cb + B * DP;                                             // [stage_rows][DP] staged queries
    float *dist = qs + (size_t)a.stage_rows * DP;                        // [R][B] distances of a round
    uint16_t *list = reinterpret_cast<uint16_t *>(dist + kPairs);       // [kListMax] queries grouped by beacon
    uint8_t *asg = reinterpret_cast<uint8_t *>(list + kListMax);         // [max_q] assignment (255: none)
    __shared__ int32_t cnt[kMaxBeacons], drawn[kMaxBeacons], first[kMaxBeacons];
    __shared__ uint8_t live[kMaxBeacons];
    __shared__ int32_t seeded_from[kMaxBeacons];                         // query seeding beacon b, or -1

    const int grp = blockIdx.x;                     // ((seq * L) + layer) * Hq + h
    const int h = grp % Hq, sl = grp / Hq, seq = sl / a.num_layers;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m = min(max(a.num_q[seq], 0), a.max_q);
    const bool staged = m <= a.stage_rows;          // else rounds are staged one at a time
    float *gb = a.beacons + (int64_t)grp * B * D;
    int32_t *gc = a.counts + (int64_t)grp * B;
    auto qidx = [&](int j, int d) -> int64_t { return (((int64_t)sl * a.max_q + j) * Hq + h) * D + d; };
    auto qval = [&](int j, int d) -> float { return staged ? qs[(size_t)j * DP + d] : load_q(a, qidx(j, d)); };

    // row-by-row copies (a warp per row, the lanes over the dimensions): no index division per element
    for (int b = warp; b < B; b += kThreads / 32)
        for (int d = lane; d < D; d += 32) cb[b * DP + d] = gb[b * D + d];
    if (staged)
        for (int j = warp; j < m; j += kThreads / 32) {
            const int64_t q0 = qidx(j, 0);
            for (int d = lane; d < D; d += 32) qs[(size_t)j * DP + d] = load_q(a, q0 + d);
        }
    if (tid < B) {
        cnt[tid] = gc[tid];
        drawn[tid] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        // 1. seeds: the j-th empty beacon takes new query j
        int t = 0;
        for (int b = 0; b < B; ++b) {
            seeded_from[b] = -1;
            if (cnt[b] > 0) {
                live[b] = 1;
            } else if (t < m) {
                seeded_from[b] = t++;
                live[b] = 1;
            } else {
                live[b] = 0;
            }
        }
    }
    __syncthreads();
    for (int b = warp; b < B; b += kThreads / 32)
        if (seeded_from[b] >= 0)
            for (int d = lane; d < D; d += 32) cb[b * DP + d] = qval(seeded_from[b], d);
    __syncthreads();

    // 2. assignment, R queries per round; each thread runs up to four distance sums side by side, every one
    // in its own fixed order
    for (int j0 = 0; j0 < m; j0 += R) {
        const int nj = min(R, m - j0);
        const float *qb = qs + (size_t)j0 * DP;
        if (!staged) {
            for (int jl = warp; jl < nj; jl += kThreads / 32) {
                const int64_t q0 = qidx(j0 + jl, 0);
                for (int d = lane; d < D; d += 32) qs[(size_t)jl * DP + d] = load_q(a, q0 + d);
            }
            qb = qs;
            __syncthreads();
        }
        const int np = nj * B;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        int qo[4], co[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = min(tid + u * kThreads, np - 1);  // lanes past the end repeat the last pair
            qo[u] = (p / B) * DP;
            co[u] = (p % B) * DP;
        }
        if (vec) {
            for (int d = 0; d < D; d += 4) {  // the same order of operations, four dimensions per load
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 x = *reinterpret_cast<const float4 *>(qb + qo[u] + d);
                    const float4 y = *reinterpret_cast<const float4 *>(cb + co[u] + d);
                    float t = __fsub_rn(x.x, y.x);
                    acc[u] = __fadd_rn(acc[u], __fmul_rn(t, t));
                    t = __fsub_rn(x.y, y.y);
                    acc[u] = __fadd_rn(acc[u], __fmul_rn(t, t));
                    t = __fsub_rn(x.z, y.z);
                    acc[u] = __fadd_rn(acc[u], __fmul_rn(t, t));
                    t = __fsub_rn(x.w, y.w);
                    acc[u] = __fadd_rn(acc[u], __fmul_rn(t, t));
                }
            }
        } else {
            for (int d = 0; d < D; ++d) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float t = __fsub_rn(qb[qo[u] + d], cb[co[u] + d]);
                    acc[u] = __fadd_rn(acc[u], __fmul_rn(t, t));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = tid + u * kThreads;
            if (p < np) dist[p] = live[p % B] ? acc[u] : INFINITY;
        }
        __syncthreads();
        for (int jl = tid; jl < nj; jl += kThreads) {
            int best = -1;
            float bd = INFINITY;
            for (int b = 0; b < B; ++b) {
                const float v = dist[jl * B + b];
                if (live[b] && (best < 0 || v < bd)) {  // strict: the lower index keeps a tie
                    best = b;
                    bd = v;
                }
            }
            asg[j0 + jl] = best < 0 ? (uint8_t)255 : (uint8_t)best;
            if (best >= 0) atomicAdd(&drawn[best], 1);
        }
        __syncthreads();
    }

    // 3. means: S = c * n, then the beacon's new queries in query order, then S / (n + drawn)
    const bool lists = m <= kListMax;
    if (lists) {
        if (tid == 0) {
            int run = 0;
            for (int b = 0; b < B; ++b) {
                first[b] = run;
                run += drawn[b];
            }
        }
        __syncthreads();
        // each warp lists its beacons' queries in ascending order (ballots over 32 queries at a time)
        for (int b = warp; b < B; b += kThreads / 32) {
            int pos = first[b];
            for (int j0 = 0; j0 < m; j0 += 32) {
                const int j = j0 + lane;
                const bool hit = j < m && asg[j] == b;
                const unsigned mask = __ballot_sync(0xffffffffu, hit);
                if (hit) list[pos + __popc(mask & ((1u << lane) - 1u))] = (uint16_t)j;
                pos += __popc(mask);
            }
        }
        __syncthreads();
    }
    for (int b = warp; b < B; b += kThreads / 32) {
        if (drawn[b] == 0) continue;  // a beacon that drew nothing keeps its value exactly
        for (int d = lane; d < D; d += 32) {
            float s = __fmul_rn(cb[b * DP + d], (float)cnt[b]);
            if (lists) {
                for (int t = 0; t < drawn[b]; ++t) s = __fadd_rn(s, qval(list[first[b] + t], d));
            } else {
                for (int j = 0; j < m; ++j)
                    if (asg[j] == b) s = __fadd_rn(s, load_q(a, qidx(j, d)));
            }
            cb[b * DP + d] = __fdiv_rn(s, (float)(cnt[b] + drawn[b]));
        }
    }
    __syncthreads();
    for (int b = warp; b < B; b += kThreads / 32)
        for (int d = lane; d < D; d += 32) gb[b * D + d] = cb[b * DP + d];
    if (tid < B) gc[tid] = cnt[tid] + drawn[tid];
    if (a.beacon_q) {
        // the beacons as the first rows of a query set [seq][layer][out_max_q][Hq][D]
        for (int b = warp; b < B; b += kThreads / 32) {
            const int64_t o0 = (((int64_t)sl * a.out_max_q + b) * Hq + h) * D;
            for (int d = lane; d < D; d += 32) {
                const float v = cb[b * DP + d];
                if (a.bf16)
                    static_cast<__nv_bfloat16 *>(a.beacon_q)[o0 + d] = __float2bfloat16_rn(v);
                else
                    static_cast<float *>(a.beacon_q)[o0 + d] = v;
            }
        }
    }
}

}  // namespace

cudaError_t launch_beacon(const void *q, const int32_t *num_q, int32_t num_seqs, int32_t num_layers,
                          int32_t num_q_heads, int32_t head_dim, int32_t max_q, bool bf16, float *beacons,
                          int32_t *counts, int32_t num_beacons, void *beacon_q, int32_t out_max_q, int32_t *status,
                          cudaStream_t stream) {
    // fixed part: beacons, a round of distances, the lists, the assignments; the rest stages queries (at
    // least one round of them, all of a group's when they fit)
    const int dp = head_dim % 4 == 0 ? head_dim + 4 : head_dim + 1;  // the kernel's padded row (DP)
    const size_t fixed = (size_t)num_beacons * dp * 4 + (size_t)kPairs * 4 + (size_t)kListMax * 2 +
                         (((size_t)max_q + 15) & ~(size_t)15);
    const int round_rows = std::min(64, kPairs / num_beacons);
    const size_t room = kSmemCap - 2048 - fixed;  // static shared memory and slack
    int rows = (int)std::min<size_t>((size_t)max_q, room / ((size_t)dp * 4));
    rows = std::max(rows, round_rows);
    const size_t smem = fixed + (size_t)rows * dp * 4;
    if (smem > kSmemCap - 2048) return cudaErrorInvalidValue;
    static int smem_set[kMaxDevices];
    cudaError_t e = dyn_smem_at_least((const void *)beacon_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    BeaconArgs a{q, num_q, num_layers, num_q_heads, head_dim, max_q, bf16 ? 1 : 0, beacons, counts, num_beacons,
                 beacon_q, out_max_q, rows, status};
    const int64_t groups = (int64_t)num_seqs * num_layers * num_q_heads;
    beacon_kernel<<<(unsigned)groups, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kvc
