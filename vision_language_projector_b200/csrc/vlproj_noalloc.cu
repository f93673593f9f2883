// Placeholder index without any allocation (declared in vlproj.h as
// vlproj_placeholder_index_noalloc).
//
// Who needs it: callers that must not allocate device memory at the point of the
// call. For example, code running where an allocation would synchronise the device
// or break a latency budget. Code that has no allocator of its own to hand, such as
// a plain C caller that only borrows buffers, needs it too. Everything else in this
// library keeps its scratch in handle-owned buffers that grow with cudaMalloc; this
// entry point needs no handle and calls no allocator.
//
// The step is the forward pass's placeholder index, the same three kernels
// (kernels_aux.cuh): per block of 4096 ids a count of placeholders, one pass that
// turns the counts into exclusive prefix sums plus their total, then every block ranks
// its own placeholders from its prefix and writes their flat positions in order. The
// per-block counts are the only scratch. Here they live in the file-scope array
// `noalloc_block_counts` below, of a fixed size that every GPU loading the library
// holds until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/vlproj.h"
#include "kernels_aux.cuh"

namespace {

constexpr int NA_MAX_BLOCKS = VLPROJ_NOALLOC_MAX_IDS / vlp::SCAN_CHUNK;      // 16384 blocks
static_assert(static_cast<int64_t>(NA_MAX_BLOCKS) * vlp::SCAN_CHUNK == VLPROJ_NOALLOC_MAX_IDS, "limit mismatch");

// The shared scratch: one count per block of ids and the total after them, one copy
// per GPU. Every call writes the entries it reads (0 .. nblocks) before reading them,
// so nothing needs clearing between calls. Calls that overlap on the same GPU (for
// example on two streams) share this array and race on it.
static __device__ __align__(256) int32_t noalloc_block_counts[NA_MAX_BLOCKS + 1];

constexpr int kMaxDevices = 64;
int32_t* g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of this device's copy of the scratch array. The host-side name of a
// __device__ array is only a stand-in, so the address comes from the runtime, once per
// device, with that device current (the first call on each device does this).
int scratch_for_current_device(int32_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VLPROJ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, noalloc_block_counts) != cudaSuccess || p == nullptr) return VLPROJ_ERR_CUDA;
        g_scratch[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch[dev];
    return VLPROJ_OK;
}

}  // namespace

extern "C" int vlproj_placeholder_index_noalloc(const int64_t* input_ids, int64_t n_ids, int64_t image_token_id,
                                                int32_t* positions, int64_t max_positions, int64_t* count,
                                                void* stream) {
    if (n_ids < 0 || n_ids > VLPROJ_NOALLOC_MAX_IDS || max_positions < 0 || count == nullptr ||
        (n_ids > 0 && input_ids == nullptr) || (max_positions > 0 && positions == nullptr))
        return VLPROJ_ERR_INVALID_ARG;
    int32_t* scratch = nullptr;
    int rc = scratch_for_current_device(&scratch);
    if (rc) return rc;
    int64_t launches = 0;
    const cudaError_t e =
        vlp::enqueue_placeholder_index(input_ids, n_ids, image_token_id, scratch, positions, max_positions, nullptr,
                                       nullptr, count, static_cast<cudaStream_t>(stream), &launches);
    return e == cudaSuccess ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}
