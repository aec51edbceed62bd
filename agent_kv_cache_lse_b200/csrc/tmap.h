// Host side of the TMA tensor maps: the driver's tiled-map encoder, resolved once, and a per-thread cache of
// the last map each call site encoded, so that a call with the same pools and shapes as the one before it
// (every round of an engine) skips the encode.  A map is a pure function of its arguments, so a cached one
// is the map the encoder would return.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstring>

namespace kvc {

enum TmapSlot { kTmapScoreK, kTmapScoreQ, kTmapLseK, kTmapLseQ, kTmapSlots };

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
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

// A bf16 map of `rank` dimensions (innermost first), unit element strides, 128-byte swizzle, 256-byte L2
// promotion, no out-of-bounds fill.  Returns CUDA_ERROR_NOT_SUPPORTED when the driver has no encoder.
inline CUresult tmap_bf16(TmapSlot slot, CUtensorMap *out, int rank, const void *addr, const cuuint64_t *dims,
                          const cuuint64_t *strides, const cuuint32_t *box) {
    struct Key {
        const void *addr;
        int rank;
        cuuint64_t dims[5], strides[4];
        cuuint32_t box[5];
    };
    struct Entry {
        bool valid;
        Key key;
        CUtensorMap map;
    };
    thread_local Entry cache[kTmapSlots] = {};
    if (rank < 1 || rank > 5) return CUDA_ERROR_INVALID_VALUE;
    Key k;
    std::memset(&k, 0, sizeof(k));
    k.addr = addr;
    k.rank = rank;
    std::memcpy(k.dims, dims, sizeof(cuuint64_t) * rank);
    std::memcpy(k.strides, strides, sizeof(cuuint64_t) * (rank - 1));
    std::memcpy(k.box, box, sizeof(cuuint32_t) * rank);
    Entry &e = cache[slot];
    if (e.valid && std::memcmp(&e.key, &k, sizeof(k)) == 0) {
        *out = e.map;
        return CUDA_SUCCESS;
    }
    auto enc = tmap_encoder();
    if (!enc) return CUDA_ERROR_NOT_SUPPORTED;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    const CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(addr), dims,
                           strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r == CUDA_SUCCESS) {
        e.valid = true;
        e.key = k;
        e.map = *out;
    } else {
        e.valid = false;
    }
    return r;
}

}  // namespace kvc
