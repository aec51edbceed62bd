// Device helpers shared by the kernels of libkvc (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kvc.h"

namespace kvc {

constexpr int kWarp = 32;

// First device error wins: status[0] = code, status[1] = row.
__device__ __forceinline__ void report(int32_t *status, int code, int row) {
    if (status == nullptr) return;
    if (atomicCAS(status, 0, code) == 0) {
        atomicExch(status + 1, row);
    }
}

// Order-preserving map of an fp32 value to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
    uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(b);
}

// Ascending int32 position -> descending-order key (larger key = smaller position).
__device__ __forceinline__ uint32_t pos_desc_key(int32_t p) {
    return ~(static_cast<uint32_t>(p) ^ 0x80000000u);
}

__device__ __forceinline__ bool is_finite(float f) {
    return (__float_as_uint(f) & 0x7f800000u) != 0x7f800000u;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// CTA-wide reductions; `red` must hold blockDim.x / 32 elements.  All threads return the result.
template <typename T>
__device__ T block_sum(T v, T *red) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    T t = lane < nw ? red[lane] : T(0);
    t = warp_sum(t);
    return t;
}

__device__ __forceinline__ float block_max(float v, float *red) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : -INFINITY;
    return warp_max(t);
}

__device__ __forceinline__ int block_or(int v, int *red) {
    return block_sum<int>(v != 0 ? 1 : 0, red) != 0;
}

// Exclusive CTA scan of an int; returns the prefix of this thread, *total gets the sum.
__device__ inline int block_exclusive_scan(int v, int *red, int *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) red[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = lane < nw ? red[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) red[lane] = s;  // inclusive per warp
    }
    __syncthreads();
    int before = (w > 0 ? red[w - 1] : 0) + x - v;
    *total = red[nw - 1];
    __syncthreads();
    return before;
}

// ---------------------------------------------------------------------------
// CTA-wide radix search over 32-bit keys, from the most significant digit down.
//
// Finds the key T at which the running weight of the keys, taken in descending key
// order, first reaches `target` (target >= 1).  weight(i) is 1 (count mode: T is the
// target-th largest key) or a non-negative fixed-point mass (mass mode).  Only
// elements with valid(i) take part.  On return (same values in every thread):
//   res.key      = T
//   res.above    = total weight of valid keys > T
//   res.eq_count = number of valid keys == T
// Digits: 11, 11, 10 bits.  Histograms live in `hcnt`/`hwt` (2048 entries each).
// Aggregation of equal digits inside a warp goes through __match_any_sync so a
// row full of equal keys does not serialise on one shared-memory atomic.
// ---------------------------------------------------------------------------

struct RadixResult {
    uint32_t key;
    unsigned long long above;
    uint32_t eq_count;
};

struct RadixShared {
    unsigned int hcnt[2048];
    unsigned long long hwt[2048];
    unsigned long long lane_w[32][32];   // per warp, per lane: weights being combined by a group leader
    uint32_t prefix, prefix_mask;
    unsigned long long above, remaining;
    uint32_t eq_count;
};

template <bool kMass, typename KeyFn, typename WeightFn, typename ValidFn>
__device__ RadixResult radix_search_desc(int n, unsigned long long target, KeyFn key, WeightFn weight,
                                         ValidFn valid, RadixShared &sh) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) {
        sh.prefix = 0;
        sh.prefix_mask = 0;
        sh.above = 0;
        sh.remaining = target;
        sh.eq_count = 0;
    }
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int b = tid; b < 2048; b += blockDim.x) {
            sh.hcnt[b] = 0;
            if (kMass) sh.hwt[b] = 0;
        }
        __syncthreads();
        const uint32_t prefix = sh.prefix, pmask = sh.prefix_mask;
        const int nround = (n + blockDim.x - 1) / blockDim.x * blockDim.x;
        for (int i = tid; i < nround; i += blockDim.x) {
            bool in = false;
            uint32_t k = 0;
            unsigned long long wv = 0;
            if (i < n && valid(i)) {
                k = key(i);
                in = (k & pmask) == prefix;
                if (kMass && in) wv = weight(i);
            }
            const unsigned active = __ballot_sync(0xffffffffu, in);
            if (in) {
                const uint32_t bin = (k >> shift) & (nb - 1);
                const unsigned peers = __match_any_sync(active, bin);
                const int leader = __ffs(peers) - 1;
                if (kMass) sh.lane_w[wid][lane] = wv;
                __syncwarp(active);
                if (lane == leader) {
                    atomicAdd(&sh.hcnt[bin], (unsigned)__popc(peers));
                    if (kMass) {
                        unsigned long long s = 0;
                        unsigned p = peers;
                        while (p) {
                            const int l = __ffs(p) - 1;
                            s += sh.lane_w[wid][l];
                            p &= p - 1;
                        }
                        atomicAdd(&sh.hwt[bin], s);
                    }
                }
                __syncwarp(active);
            }
        }
        __syncthreads();
        // warp 0: walk bins from the top until the running weight reaches `remaining`
        if (tid < 32) {
            const int per = nb / 32;
            const int hi = nb - 1 - lane * per;  // this lane covers bins hi, hi-1, ..., hi-per+1
            unsigned long long mine = 0;
            for (int b = 0; b < per; ++b) {
                const int bin = hi - b;
                mine += kMass ? sh.hwt[bin] : (unsigned long long)sh.hcnt[bin];
            }
            // inclusive scan over lanes (lane 0 = top bins)
            unsigned long long incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned long long excl = incl - mine;
            const unsigned long long rem = sh.remaining;
            const bool here = excl < rem && incl >= rem;
            const unsigned who = __ballot_sync(0xffffffffu, here);
            if (here && lane == __ffs(who) - 1) {
                unsigned long long run = excl;
                for (int b = 0; b < per; ++b) {
                    const int bin = hi - b;
                    const unsigned long long w = kMass ? sh.hwt[bin] : (unsigned long long)sh.hcnt[bin];
                    if (run + w >= rem) {
                        sh.above += run;
                        sh.remaining = rem - run;
                        sh.prefix |= (uint32_t)bin << shift;
                        sh.prefix_mask |= (uint32_t)(nb - 1) << shift;
                        sh.eq_count = sh.hcnt[bin];
                        break;
                    }
                    run += w;
                }
            }
        }
        __syncthreads();
    }
    RadixResult r;
    r.key = sh.prefix;
    r.above = sh.above;
    r.eq_count = sh.eq_count;
    __syncthreads();
    return r;
}

}  // namespace kvc
