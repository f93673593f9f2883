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
// The step is the same as the forward pass's placeholder index: per block of 4096
// ids a count of placeholders, then every block ranks its own placeholders from the
// counts of the blocks before it and writes their flat positions in order. The
// per-block counts are the only scratch. Here they live in the file-scope array
// `noalloc_block_counts` below, of a fixed size that every GPU loading the library
// holds until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/vlproj.h"

namespace {

constexpr int NA_THREADS = 256;
constexpr int NA_ITEMS = 16;
constexpr int NA_CHUNK = NA_THREADS * NA_ITEMS;                       // ids per block
constexpr int NA_MAX_BLOCKS = VLPROJ_NOALLOC_MAX_IDS / NA_CHUNK;      // 16384 blocks
static_assert(static_cast<int64_t>(NA_MAX_BLOCKS) * NA_CHUNK == VLPROJ_NOALLOC_MAX_IDS, "limit mismatch");

// The shared scratch: one count per block of ids, one copy per GPU. Every call writes
// the entries it reads (blocks 0 .. nblocks-1) before reading them, so nothing needs
// clearing between calls. Calls that overlap on the same GPU (for example on two
// streams) share this array and race on it.
static __device__ __align__(256) int32_t noalloc_block_counts[NA_MAX_BLOCKS];

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

__device__ __forceinline__ int na_block_sum(int v, int* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < NA_THREADS / 32; ++w) t += red[w];
    return t;
}

// counts[b] = placeholders among ids[b*NA_CHUNK, (b+1)*NA_CHUNK)
__global__ void __launch_bounds__(NA_THREADS) vlp_na_count_kernel(const int64_t* __restrict__ ids, int64_t n,
                                                                  int64_t token, int32_t* __restrict__ counts) {
    __shared__ int red[NA_THREADS / 32];
    const int64_t start = static_cast<int64_t>(blockIdx.x) * NA_CHUNK;
    int c = 0;
#pragma unroll
    for (int i = 0; i < NA_ITEMS; ++i) {
        const int64_t idx = start + i * NA_THREADS + threadIdx.x;
        if (idx < n && __ldg(&ids[idx]) == token) ++c;
    }
    c = na_block_sum(c, red);
    if (threadIdx.x == 0) counts[blockIdx.x] = c;
}

// positions[j] = flat index of the j-th placeholder (j < max_pos); *count = total.
__global__ void __launch_bounds__(NA_THREADS) vlp_na_compact_kernel(const int64_t* __restrict__ ids, int64_t n,
                                                                    int64_t token, const int32_t* __restrict__ counts,
                                                                    int nblocks, int32_t* __restrict__ positions,
                                                                    int64_t max_pos, int64_t* __restrict__ count) {
    __shared__ int red[NA_THREADS / 32];
    __shared__ int warp_cnt[NA_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int pre = 0, tot = 0;
    for (int b = threadIdx.x; b < nblocks; b += NA_THREADS) {
        const int c = counts[b];
        tot += c;
        if (b < static_cast<int>(blockIdx.x)) pre += c;
    }
    pre = na_block_sum(pre, red);
    tot = na_block_sum(tot, red);
    if (blockIdx.x == 0 && threadIdx.x == 0) *count = tot;
    const int64_t start = static_cast<int64_t>(blockIdx.x) * NA_CHUNK;
    int64_t run = pre;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i = 0; i < NA_ITEMS; ++i) {
        const int64_t idx = start + i * NA_THREADS + threadIdx.x;
        const bool flag = idx < n && __ldg(&ids[idx]) == token;
        const unsigned bal = __ballot_sync(0xffffffffu, flag);
        if (lane == 0) warp_cnt[warp] = __popc(bal);
        __syncthreads();
        int before = 0, all = 0;
#pragma unroll
        for (int w = 0; w < NA_THREADS / 32; ++w) {
            const int c = warp_cnt[w];
            before += (w < warp) ? c : 0;
            all += c;
        }
        const int64_t rank = run + before + __popc(bal & lt_mask);
        if (flag && rank < max_pos) positions[rank] = static_cast<int32_t>(idx);
        run += all;
        __syncthreads();
    }
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nblocks = static_cast<int>((n_ids + NA_CHUNK - 1) / NA_CHUNK);
    if (nblocks > 0) vlp_na_count_kernel<<<nblocks, NA_THREADS, 0, s>>>(input_ids, n_ids, image_token_id, scratch);
    vlp_na_compact_kernel<<<nblocks > 0 ? nblocks : 1, NA_THREADS, 0, s>>>(
        input_ids, n_ids, image_token_id, scratch, nblocks, positions, max_positions, count);
    return cudaGetLastError() == cudaSuccess ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}
