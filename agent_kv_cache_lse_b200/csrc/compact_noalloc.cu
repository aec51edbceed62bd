// kvc_compact_pages_noalloc: the compaction entry point for callers that cannot allocate.
//
// kvc_compact_pages needs a small device workspace (one 64-bit offset per row) for the
// freed-page list.  Some callers have no way to provide one: serving engines whose
// allocator has already handed the whole device to the KV pool, or plugins that
// reach this library through a foreign-function boundary without access to the host
// framework's allocator.  This variant keeps the workspace in a fixed array in the
// library's own device memory instead, so the caller passes only the cache, the plan
// and the outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// it (kNoAllocMaxRows + 1 int64 values, 128 KiB) until the process exits.  Host code
// cannot use the array's name as a device address, so the first call on each device
// looks the address up with cudaGetSymbolAddress (with that device current) and caches
// it.  All calls
// share the array: calls whose kernels overlap on the GPU (for instance on two streams)
// race on it and must be serialised by the caller.  Nothing in it needs to start at
// zero: the offset kernel writes every entry it later reads.
#include <mutex>

#include "../../include/kvc.h"
#include "internal.h"

namespace {

constexpr int kNoAllocMaxRows = KVC_NOALLOC_MAX_ROWS;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int64_t g_noalloc_offsets[kNoAllocMaxRows + 1];

std::mutex g_setup_mutex;
int64_t *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device (looked up once per device).
cudaError_t scratch_on_current_device(int64_t **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_offsets);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<int64_t *>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kvc_status kvc_compact_pages_noalloc(const kvc_cache *cache, const int32_t *move_src,
                                                const int32_t *move_dst, const int32_t *num_moves,
                                                const int32_t *new_len, float *crf, int32_t *freed,
                                                int64_t freed_capacity, int64_t *num_freed, int32_t *d_status,
                                                kvc_stream_t stream) {
    if (cache && (int64_t)cache->num_seqs * cache->num_layers * cache->num_kv_heads > kNoAllocMaxRows) {
        kvc::set_last_error("kvc_compact_pages_noalloc supports at most %d rows (KVC_NOALLOC_MAX_ROWS)",
                            kNoAllocMaxRows);
        return KVC_ERR_UNSUPPORTED;
    }
    int64_t *scratch = nullptr;
    cudaError_t e = scratch_on_current_device(&scratch);
    if (e != cudaSuccess) {
        kvc::set_last_error("kvc_compact_pages_noalloc: device address of the built-in workspace: %s",
                            cudaGetErrorString(e));
        return KVC_ERR_CUDA;
    }
    // the regular entry point's checks and launches, with the library's own array as the workspace
    return kvc_compact_pages(cache, move_src, move_dst, num_moves, new_len, crf, freed, freed_capacity, num_freed,
                             scratch, (size_t)(kNoAllocMaxRows + 1) * sizeof(int64_t), d_status, stream);
}
