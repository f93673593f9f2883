// Host-side pieces shared by the library's translation units: driver entry points,
// tensor-map encoders, device scratch buffers, the batch plan (closed-form geometry),
// GEMM launchers, and the handle behind the opaque vlproj_handle.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/vlproj.h"
#include "gemm_sm100.cuh"
#include "kernels_aux.cuh"

#define VLP_CUDA(call)                                                                        \
    do {                                                                                      \
        cudaError_t e_ = (call);                                                              \
        if (e_ != cudaSuccess) {                                                              \
            std::fprintf(stderr, "vlproj: %s failed: %s (%s:%d)\n", #call, cudaGetErrorString(e_), \
                         __FILE__, __LINE__);                                                 \
            return VLPROJ_ERR_CUDA;                                                           \
        }                                                                                     \
    } while (0)

namespace vlp_host {

using vlp::GemmLayout;
using vlp::GemmParams;
using vlp::ImageDesc;
using vlp::ViewDesc;


constexpr uint64_t kDefaultWaitNs = 2000000000ull;
// Tile queues per handle (dynamic tile order): counter pairs taken in turn by launches.
constexpr uint32_t kTileQueues = 64;
// Automatic tile order: GEMMs whose A is a plain row-major matrix keep the static order
// below this much work, counted in waves of 64-K-block tiles (measured 1-3 % slower in the
// dynamic order at 10-25 such waves: MoonViT's GEMM1 over the merged copy, VL2's and
// DS-ViT's GEMM2, MoonViT's weight gradients); the rest take the dynamic one (1-2 % faster
// for the gathered-A GEMM1s; on the Stress batch under the power cap, 300-600 such waves,
// 11 % for the forward, where it halves the DRAM reads, and 6 % for the backward).
constexpr int kDynamicMinWaves = 64;

struct DriverFns {
    PFN_cuTensorMapEncodeTiled_v12000 tiled = nullptr;
    PFN_cuTensorMapEncodeIm2col_v12000 im2col = nullptr;
};

inline const DriverFns& driver() {
    static DriverFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeIm2col", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.im2col = reinterpret_cast<PFN_cuTensorMapEncodeIm2col_v12000>(p);
    });
    return fns;
}

// 2D bf16 row-major matrix [rows][cols] with row stride ld elements (0 = cols, a
// multiple of 8), box = box_rows x 64 columns, 128-byte swizzle, out-of-range elements
// read as zero.
inline int encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                          uint64_t ld = 0) {
    auto fn = driver().tiled;
    if (!fn) return VLPROJ_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {(ld ? ld : cols) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(vlp::BK), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}

// Output map of a bf16 matrix [rows][cols] with row stride ld elements (0 = cols, a
// multiple of 8) for the TMA-store epilogues: 32 x 32 boxes, no swizzle; boxes reaching
// past the matrix are clipped.
inline int encode_bf16_store(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld = 0) {
    auto fn = driver().tiled;
    if (!fn) return VLPROJ_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {(ld ? ld : cols) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}

// Map of a row-major bf16 matrix [rows][cols] (cols a multiple of 64) read as the
// MN-major operand of a GEMM whose K runs over its rows: seen as 3D (c % 64, r, c / 64),
// a box (64, 64, strips) holds 64 rows of `strips` 64-column strips, each strip 8 KB
// contiguous in shared memory with the 128-byte swizzle (the canonical MN-major layout).
// Rows past `rows` read as zeros.
inline int encode_bf16_mn(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t strips) {
    auto fn = driver().tiled;
    if (!fn || cols % 64) return VLPROJ_ERR_CUDA;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(vlp::BK), strips};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}

// im2col map of n views of one (h, w) grid of C-channel bf16 patches, packed back to
// back from `base`: the k x k, stride-k window walk of the merge. Base positions run
// over 0, k, ..., k*(w'-1) (lower corner 0, upper corner k*w' - w - (k-1), the
// convolution form of "pad the high end to k*w'"), `pixels` per load, 64 channels each.
inline int encode_im2col(CUtensorMap* map, const void* base, int C, int h, int w, int n, int k, int pixels) {
    auto fn = driver().im2col;
    if (!fn) return VLPROJ_ERR_CUDA;
    const int hp = (h + k - 1) / k, wp = (w + k - 1) / k;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(w), static_cast<cuuint64_t>(h),
                          static_cast<cuuint64_t>(n)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(w) * C * 2,
                             static_cast<cuuint64_t>(h) * w * C * 2};
    int lower[2] = {0, 0};
    int upper[2] = {k * wp - w - (k - 1), k * hp - h - (k - 1)};
    cuuint32_t estr[4] = {1, static_cast<cuuint32_t>(k), static_cast<cuuint32_t>(k), 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, lower, upper,
                    static_cast<cuuint32_t>(vlp::BK), static_cast<cuuint32_t>(pixels), estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}

// 5D tiled map of n views of one (h, w) grid with k | h, k | w and w' | 128: dims
// (C, k, w', k, h' * n) with strides (C, k*C, w*C, k*w*C) elements, box
// (64, 1, w', 1, 128 / w'): one box is 128 merged tokens, row-major, at filter tap
// (dy, dx) = (coordinate 3, coordinate 1).
inline int encode_box5(CUtensorMap* map, const void* base, int C, int h, int w, int n, int k) {
    auto fn = driver().tiled;
    if (!fn) return VLPROJ_ERR_CUDA;
    const int hp = h / k, wp = w / k;
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(wp),
                          static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(hp) * n};
    const cuuint64_t e = 2;
    cuuint64_t strides[4] = {static_cast<cuuint64_t>(C) * e, static_cast<cuuint64_t>(k) * C * e,
                             static_cast<cuuint64_t>(w) * C * e, static_cast<cuuint64_t>(k) * w * C * e};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(vlp::BK), 1, static_cast<cuuint32_t>(wp), 1,
                         static_cast<cuuint32_t>(vlp::BM / wp)};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VLPROJ_OK : VLPROJ_ERR_CUDA;
}

template <typename T>
struct DevBuf {
    T* ptr = nullptr;
    size_t cap = 0;   // elements
    int ensure(size_t n) {
        if (n <= cap) return VLPROJ_OK;
        if (ptr) cudaFree(ptr);
        ptr = nullptr;
        cap = 0;
        size_t want = std::max<size_t>(n, 1) + n / 4;
        if (cudaMalloc(&ptr, want * sizeof(T)) != cudaSuccess) return VLPROJ_ERR_CUDA;
        cap = want;
        return VLPROJ_OK;
    }
    void release() {
        if (ptr) cudaFree(ptr);
        ptr = nullptr;
        cap = 0;
    }
};

// Pinned host staging for small per-call uploads: reused only after the previous
// copy out of it has executed; skipped when the bytes equal the last upload.
struct Uploader {
    uint8_t* staging = nullptr;
    size_t cap = 0;
    cudaEvent_t done = nullptr;
    std::vector<uint8_t> last;
    bool valid = false;
    int put(void* dst, const void* src, size_t bytes, cudaStream_t s) {
        if (valid && last.size() == bytes && std::memcmp(last.data(), src, bytes) == 0) {
            // unchanged: the device copy is (or will be) there; order `s` after it
            if (done && bytes) VLP_CUDA(cudaStreamWaitEvent(s, done, 0));
            return VLPROJ_OK;
        }
        valid = false;
        if (bytes == 0) return VLPROJ_OK;
        if (!done) VLP_CUDA(cudaEventCreateWithFlags(&done, cudaEventDisableTiming));
        VLP_CUDA(cudaEventSynchronize(done));
        if (bytes > cap) {
            if (staging) cudaFreeHost(staging);
            staging = nullptr;
            cap = 0;
            VLP_CUDA(cudaMallocHost(&staging, bytes * 2));
            cap = bytes * 2;
        }
        std::memcpy(staging, src, bytes);
        VLP_CUDA(cudaMemcpyAsync(dst, staging, bytes, cudaMemcpyHostToDevice, s));
        VLP_CUDA(cudaEventRecord(done, s));
        last.assign(static_cast<const uint8_t*>(src), static_cast<const uint8_t*>(src) + bytes);
        valid = true;
        return VLPROJ_OK;
    }
    void invalidate() { valid = false; }
    void release() {
        if (done) cudaEventSynchronize(done);
        if (staging) cudaFreeHost(staging);
        if (done) cudaEventDestroy(done);
        staging = nullptr;
        done = nullptr;
        cap = 0;
        valid = false;
    }
};

struct Plan {
    std::vector<ViewDesc> views;
    std::vector<ImageDesc> images;
    int64_t M = 0;          // GEMM rows (merged tokens, varlen im2col runs padded to `chunk`)
    int64_t M_real = 0;     // merged tokens
    int64_t R = 0;          // assembled rows
    int64_t P = 0;          // patches
    int max_special = 0;    // most special rows of one image
    bool uniform = true;    // every view has the same grid
    bool im2col = true;     // GEMM1 gathers with TMA im2col (else cp.async)
    bool box5 = false;      // ... or with one 5D tiled box per K-block (regular grids)
    bool merged_ln = false; // ... or reads A written in token order by the LayerNorm pass
    bool fused = false;     // ... or produces A inside GEMM1 (merge + LayerNorm / convert)
    bool tgather = false;   // ... or gathers A by 128 threads' cp.async (CTA pairs allowed)
    bool tgather_ln = false;// ... and applies the LayerNorm to it in shared memory
    int chunk = 128;        // im2col rows per load
};

inline int validate_config(const vlproj_config* c) {
    if (!c) return VLPROJ_ERR_INVALID_ARG;
    if (c->depth < 2 || c->depth > 8 || c->tile_tag == VLPROJ_TILE_1D || c->token_pooling != 0)
        return VLPROJ_ERR_UNSUPPORTED;
    if (c->k < 1 || c->k > 3) return VLPROJ_ERR_UNSUPPORTED;
    if (c->tile_tag != VLPROJ_TILE_NONE && c->tile_tag != VLPROJ_TILE_2D) return VLPROJ_ERR_UNSUPPORTED;
    if (c->global_view_pos != VLPROJ_GLOBAL_HEAD && c->global_view_pos != VLPROJ_GLOBAL_TAIL)
        return VLPROJ_ERR_INVALID_ARG;
    if (c->feat_dtype != VLPROJ_FEAT_BF16 && c->feat_dtype != VLPROJ_FEAT_F32) return VLPROJ_ERR_INVALID_ARG;
    if (c->k_order != VLPROJ_ORDER_CHANNEL_OUTER && c->k_order != VLPROJ_ORDER_POSITION_OUTER)
        return VLPROJ_ERR_INVALID_ARG;
    if (c->C <= 0 || c->C % 64 != 0 || c->N1 <= 0 || c->N1 % 64 != 0 || c->N2 <= 0 || c->N2 % 32 != 0)
        return VLPROJ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(c->k) * c->k * c->C > (1 << 20) || c->N1 > (1 << 20) || c->N2 > (1 << 20))
        return VLPROJ_ERR_INVALID_ARG;
    return VLPROJ_OK;
}

// Closed-form geometry of one batch. Returns an error for inconsistent shapes.
// gather_mode (VLPROJ_GATHER_*) resolves to im2col or cp.async here (plan.im2col);
// with im2col and views of different grids each view's run of GEMM rows is padded to
// a multiple of 32, so the im2col loads of per-view maps never straddle two views.
inline int build_plan(const vlproj_config& c, const int32_t* grid_hw, const int32_t* crop, int32_t n_images,
               bool tiled_override_none, int gather_mode, Plan* out) {
    Plan& pl = *out;
    pl = Plan();
    if (n_images < 0) return VLPROJ_ERR_INVALID_ARG;
    if (n_images > 0 && !grid_hw) return VLPROJ_ERR_INVALID_ARG;
    const bool tiled = !tiled_override_none && c.tile_tag == VLPROJ_TILE_2D;
    if (tiled && n_images > 0 && !crop) return VLPROJ_ERR_INVALID_ARG;
    const int k = c.k;
    // first pass: view count, shapes, uniformity
    int64_t n_views = 0;
    for (int32_t img = 0; img < n_images; ++img) {
        const int tw = tiled ? crop[2 * img] : 0;
        const int th = tiled ? crop[2 * img + 1] : 0;
        if (tiled && (tw < 1 || th < 1 || static_cast<int64_t>(tw) * th > 4096)) return VLPROJ_ERR_INVALID_ARG;
        n_views += tiled ? 1 + tw * th : 1;
    }
    for (int64_t v = 0; v < n_views; ++v) {
        const int h = grid_hw[2 * v], w = grid_hw[2 * v + 1];
        if (h < 1 || w < 1 || h > 65535 || w > 65535) return VLPROJ_ERR_INVALID_ARG;
        if (h != grid_hw[0] || w != grid_hw[1]) pl.uniform = false;
    }
    pl.chunk = pl.uniform ? 128 : 32;
    const bool f32 = c.feat_dtype == VLPROJ_FEAT_F32;
    if ((gather_mode == VLPROJ_GATHER_AUTO && (c.has_ln || f32)) || gather_mode == VLPROJ_GATHER_MERGED) {
        // a LayerNorm / convert pass writes a bf16 copy anyway: write it as A itself,
        // already merged, so GEMM1 reads a plain matrix by TMA tiles (measured faster than
        // normalising inside GEMM1 behind the thread gather)
        pl.merged_ln = true;
        pl.im2col = false;
        gather_mode = VLPROJ_GATHER_CPASYNC;   // no padding, no chunk table
    } else if (gather_mode == VLPROJ_GATHER_FUSED) {
        // the same copy, written by GEMM1's own producer warps just ahead of its TMA loads
        pl.fused = true;
        pl.im2col = false;
        gather_mode = VLPROJ_GATHER_CPASYNC;
    } else if (gather_mode == VLPROJ_GATHER_THREADS) {
        // GEMM1 gathers the raw patches itself and, with a LayerNorm on bf16 features,
        // normalises them in shared memory (only the per-patch statistics go through
        // memory); with fp32 features a convert / LayerNorm pass runs first
        pl.tgather = true;
        pl.tgather_ln = c.has_ln && !f32;
        pl.im2col = false;
        gather_mode = VLPROJ_GATHER_CPASYNC;
    }
    pl.im2col = !pl.merged_ln && !pl.tgather && !pl.fused &&
                (gather_mode == VLPROJ_GATHER_IM2COL || (gather_mode == VLPROJ_GATHER_AUTO && pl.uniform));
    if (pl.uniform && n_views > 0 && !pl.fused && !pl.merged_ln && !pl.tgather &&
        (gather_mode == VLPROJ_GATHER_BOX || gather_mode == VLPROJ_GATHER_AUTO)) {
        const int h = grid_hw[0], w = grid_hw[1];
        if (h % k == 0 && w % k == 0 && w / k <= vlp::BM && vlp::BM % (w / k) == 0) {
            pl.box5 = true;
            pl.im2col = false;
        } else if (gather_mode == VLPROJ_GATHER_BOX) {
            pl.im2col = true;             // not regular: the im2col walk does the same job
        }
    }
    const int pad_to = (pl.im2col && !pl.uniform) ? pl.chunk : 1;
    int64_t v = 0;
    for (int32_t img = 0; img < n_images; ++img) {
        const int tw = tiled ? crop[2 * img] : 0;
        const int th = tiled ? crop[2 * img + 1] : 0;
        const int nv = tiled ? 1 + tw * th : 1;
        const int h0 = grid_hw[2 * v], w0 = grid_hw[2 * v + 1];
        const int hp = (h0 + k - 1) / k, wp = (w0 + k - 1) / k;
        int64_t rows;
        if (tiled)
            rows = static_cast<int64_t>(hp) * (wp + 1) + 1 +
                   static_cast<int64_t>(th) * hp * (static_cast<int64_t>(tw) * wp + 1);
        else
            rows = static_cast<int64_t>(hp) * wp;
        for (int t = 0; t < nv; ++t, ++v) {
            const int h = grid_hw[2 * v], w = grid_hw[2 * v + 1];
            if (h != h0 || w != w0) return VLPROJ_ERR_INVALID_ARG;   // views of one image share a grid
            ViewDesc d{};
            d.patch_start = pl.P;
            d.tok_start = static_cast<int32_t>(pl.M);
            d.tok_real = static_cast<int32_t>(pl.M_real);
            d.h = h; d.w = w; d.hp = hp; d.wp = wp;
            d.row_base = static_cast<int32_t>(pl.R);
            d.view_in_image = t;
            d.tw = tw; d.th = th;
            d.tail = tiled && c.global_view_pos == VLPROJ_GLOBAL_TAIL;
            pl.views.push_back(d);
            const int64_t toks = static_cast<int64_t>(hp) * wp;
            pl.P += static_cast<int64_t>(h) * w;
            pl.M_real += toks;
            pl.M += (toks + pad_to - 1) / pad_to * pad_to;
            if (pl.P >= (int64_t(1) << 31) || pl.M >= (int64_t(1) << 30)) return VLPROJ_ERR_INVALID_ARG;
        }
        if (tiled) {
            ImageDesc im{};
            im.row_base = static_cast<int32_t>(pl.R);
            im.hp = hp; im.wp = wp; im.tw = tw; im.th = th;
            im.tail = c.global_view_pos == VLPROJ_GLOBAL_TAIL;
            pl.images.push_back(im);
            pl.max_special = std::max(pl.max_special, hp + th * hp + 1);
        }
        pl.R += rows;
        if (pl.R >= (int64_t(1) << 31)) return VLPROJ_ERR_INVALID_ARG;
    }
    return VLPROJ_OK;
}

// N-blocks per raster band: all of them while B fits in about half of the 126 MB L2
// (64 MB), else the fewest bands under that budget, of equal width, so that no band is
// a narrow remainder whose tiles share little of A.
// When even one N-block's slice of B is larger than the default budget (the weight
// gradients, where K is the batch's token count), no band stays in L2 and the operands
// stream from memory in panels: then bands of about sqrt(units) N-blocks make the units
// running together read the fewest panels (units M-blocks x N-blocks in one wave), instead
// of one N-block against every M-block. An explicit budget keeps the plain rule.
inline int raster_group(int N, int K, int BN, int64_t budget = 0, int units = 74) {
    const int n_tiles = (N + BN - 1) / BN;
    const int64_t per_block = static_cast<int64_t>(BN) * K * 2;
    if (budget <= 0) {
        budget = int64_t(64) << 20;
        if (per_block > budget) {
            const int g = static_cast<int>(std::lround(std::sqrt(static_cast<double>(std::max(units, 1)))));
            return std::max(1, std::min(n_tiles, g));
        }
    }
    const int max_group = static_cast<int>(std::max<int64_t>(1, budget / per_block));
    if (n_tiles <= max_group) return n_tiles;
    const int bands = (n_tiles + max_group - 1) / max_group;
    return (n_tiles + bands - 1) / bands;
}

template <int BN, int A, int E, int CTAS>
int launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const CUtensorMap& tc2,
                GemmParams p, int num_sms, cudaStream_t s) {
    using L = GemmLayout<BN, CTAS, vlp::epi_stage_bytes(E) * vlp::epi_groups(BN), vlp::a_aux_bytes(A)>;
    auto kernel = vlp::vlp_gemm_kernel<BN, A, E, CTAS>;
    if (p.group_n <= 0) p.group_n = raster_group(p.N, p.K, BN, p.l2_budget, num_sms / CTAS);
    VLP_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_ALLOC));
    const int tiles = ((p.M + vlp::BM * CTAS - 1) / (vlp::BM * CTAS)) * ((p.N + BN - 1) / BN);
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(vlp::gemm_threads(A, BN));
    cfg.dynamicSmemBytes = L::SMEM_ALLOC;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CTAS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    int resident = num_sms / CTAS;               // persistent: one unit per SM (pair of SMs)
    if constexpr (CTAS > 1) {
        // pairs must sit in one GPC: ask how many can be resident at once
        static int cached = -1;
        if (cached < 0) {
            cfg.gridDim = dim3(static_cast<unsigned>(2 * resident));
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            cached = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess && n > 0 ? n : resident;
        }
        resident = std::min(resident, cached);
    }
    const int units = std::min(tiles, resident);
    if (units <= 0) return VLPROJ_OK;
    cfg.gridDim = dim3(static_cast<unsigned>(units * CTAS));
    cfg.attrs = CTAS > 1 ? attr : nullptr;
    cfg.numAttrs = CTAS > 1 ? 1 : 0;
    VLP_CUDA(cudaLaunchKernelEx(&cfg, kernel, ta, tb, tc, tc2, p));
    return VLPROJ_OK;
}

inline int pick_bn(int N) { return N >= 256 ? 256 : 128; }

}  // namespace vlp_host

// The state behind the opaque handle: copies of the weights, their tensor maps, and
// scratch buffers that grow on demand and are kept between calls.
struct vlproj_handle {
    vlproj_config cfg{};
    int device = 0;
    int num_sms = 148;
    int K1 = 0;
    uint64_t wait_ns = vlp_host::kDefaultWaitNs;
    int gather_mode = VLPROJ_GATHER_AUTO;
    __nv_bfloat16* W1p = nullptr;
    __nv_bfloat16* W2 = nullptr;
    float* b1 = nullptr;
    float* b2 = nullptr;
    float* gamma = nullptr;
    float* beta = nullptr;
    CUtensorMap tmW1{}, tmW2{};          // B boxes of BN rows (single-CTA tiles)
    CUtensorMap tmW1h{}, tmW2h{};        // B boxes of 128 rows (each CTA of a pair loads half)
    bool pairs = true;                   // run 256 x 256 tiles on CTA pairs where possible
    int64_t l2_budget = 0;               // forward GEMMs: bytes of B per raster band (0 = 64 MB)
    // dynamic tile order: kTileQueues counter pairs, taken in turn by successive GEMM
    // launches (kernels that may overlap, on the caller's and the side stream, are a few
    // launches apart and so never share one)
    int tile_order = VLPROJ_TILE_ORDER_AUTO;
    int* tqueue = nullptr;
    uint32_t tq_next = 0;
    // scratch, grown on demand
    vlp_host::DevBuf<__nv_bfloat16> H, H2, Xn, A;       // H2: second hidden buffer (depth > 2)
    // middle layers (depth > 2): weights, biases, tensor maps (BN-row and 128-row boxes)
    std::vector<__nv_bfloat16*> Wm;
    std::vector<float*> bm;
    std::vector<CUtensorMap> tmWm, tmWmh;
    vlp_host::DevBuf<int32_t> pos, rowdest, counts;
    vlp_host::DevBuf<int2> gmeta;
    vlp_host::DevBuf<float2> lnstats;    // per (tap, GEMM row) LayerNorm statistics (A_TGATHER_LN)
    vlp_host::DevBuf<uint32_t> fwork;    // A_FUSED: item counter (64-bit) and per (block, tap) counters
    vlp_host::DevBuf<int4> chunks;
    vlp_host::DevBuf<vlp::ViewDesc> dviews;
    vlp_host::DevBuf<vlp::ImageDesc> dimages;
    vlp_host::DevBuf<CUtensorMap> dmaps;
    int* status = nullptr;       // [0] latched error, [1] per-forward count check
    int lnp_per_sm = 0;          // resident blocks per SM of the LayerNorm-merge kernel (0: not queried)
    vlp_host::Uploader up_views, up_images, up_maps;
    std::vector<CUtensorMap> host_maps;
    // the placeholder index runs on `side`, forked from / joined to the caller's stream
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr, join2 = nullptr;
    // tracing: start / end event of every stage, recorded on the stream that runs it
    bool profiling = false;
    uint32_t profile_mask = ~0u;         // stages that record events while profiling
    bool profiled_valid = false;
    cudaEvent_t ev_begin[VLPROJ_NUM_STAGES] = {};
    cudaEvent_t ev_end[VLPROJ_NUM_STAGES] = {};
    bool stage_ran[VLPROJ_NUM_STAGES] = {};
    int64_t launches = 0;
    // cached tensor map of H
    CUtensorMap tmH{};
    const void* tmH_ptr = nullptr;
    int64_t tmH_rows = -1;
    // backward: transposed weights (made on the first backward call) and scratch
    __nv_bfloat16* W2t = nullptr;        // [N1][N2]
    __nv_bfloat16* W1pt = nullptr;       // [K1][N1], rows in position-outer order
    CUtensorMap tmW2t{}, tmW2th{}, tmW1pt{}, tmW1pth{};
    std::vector<__nv_bfloat16*> Wmt;     // middle layers transposed, [N1][N1] each
    std::vector<CUtensorMap> tmWmt, tmWmth;
    // G, Hr: GELU'(P) and H, one [M][N1] slab each per hidden layer; dP: two slabs, layer
    // by layer; dY [M][N2]; dW1p: dW1 in the kernel's K order before it is reordered
    vlp_host::DevBuf<__nv_bfloat16> G, Hr, dY, dP;
    vlp_host::DevBuf<float> dW1p;
    vlp_host::DevBuf<float> part_cs;     // column-sum partials of the bias gradients
    vlp_host::DevBuf<__nv_bfloat16> dA;
    vlp_host::DevBuf<float> part, part_sp;
    // host-memory entry point: copy streams, per-slot events and double-buffered staging
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};
    vlp_host::DevBuf<uint8_t> stage_feat[2];
    vlp_host::DevBuf<__nv_bfloat16> stage_rows[2];
};

namespace vlp_host {

// Tile shape: 256 x 256 tiles on CTA pairs when N allows and the A operand comes by
// TMA; 128 x 256 (or x 128 for N < 256) on single CTAs otherwise. tc / tc2: output
// maps of the TMA-store epilogues (unused by the others). A launch in the dynamic tile
// order takes the handle's next tile queue.
inline const CUtensorMap& no_map() {
    static const CUtensorMap zero{};
    return zero;
}

template <int A, int E>
int launch_gemm_bn(vlproj_handle* h, int bn, bool pair, const CUtensorMap& ta, const CUtensorMap& tb,
                   const CUtensorMap& tb_half, GemmParams p, cudaStream_t s, const CUtensorMap& tc = no_map(),
                   const CUtensorMap& tc2 = no_map()) {
    const int num_sms = h->num_sms;
    const int ctas = (A != vlp::A_CPASYNC && pair && bn >= 256) ? 2 : 1;
    const int64_t tiles = ((static_cast<int64_t>(p.M) + vlp::BM * ctas - 1) / (vlp::BM * ctas)) * ((p.N + bn - 1) / bn);
    const int64_t kblocks = (static_cast<int64_t>(p.K) + vlp::BK - 1) / vlp::BK;
    const bool dyn = h->tile_order == VLPROJ_TILE_ORDER_DYNAMIC ||
                     (h->tile_order == VLPROJ_TILE_ORDER_AUTO &&
                      (A != vlp::A_TILE ||
                       tiles * kblocks >= static_cast<int64_t>(kDynamicMinWaves) * 64 * (num_sms / ctas)));
    p.tile_queue = (dyn && h->tqueue) ? h->tqueue + 2 * (h->tq_next++ % kTileQueues) : nullptr;
    if constexpr (A == vlp::A_IM2COL && E == vlp::EPI_GELU) {
        if (pair && bn == 512) return launch_gemm<512, A, E, 2>(ta, tb_half, tc, tc2, p, num_sms, s);
    }
    if constexpr (A != vlp::A_CPASYNC) {
        if (pair && bn >= 256) return launch_gemm<256, A, E, 2>(ta, tb_half, tc, tc2, p, num_sms, s);
    }
    if (bn >= 256) return launch_gemm<256, A, E, 1>(ta, tb, tc, tc2, p, num_sms, s);
    return launch_gemm<128, A, E, 1>(ta, tb, tc, tc2, p, num_sms, s);
}

// Stage timing: begin / end events on the stream that runs the stage.
inline void stage_begin(vlproj_handle* h, int stage, cudaStream_t s) {
    h->stage_ran[stage] = ((h->profile_mask >> stage) & 1u) != 0;
    if (h->profiling && ((h->profile_mask >> stage) & 1u)) cudaEventRecord(h->ev_begin[stage], s);
}
inline void stage_end(vlproj_handle* h, int stage, cudaStream_t s) {
    if (h->profiling && ((h->profile_mask >> stage) & 1u)) cudaEventRecord(h->ev_end[stage], s);
}

// LayerNorm-merge launch: the pipelined form when C fits (C <= 2048), a grid of the
// blocks that fit on the SMs at once, each warp with a ring of about 9 KB of patch rows
// (2 to 16 rows; MoonViT's 2304-byte rows: 4 per warp, 2 blocks per SM, measured
// faster than 3 rows at 3 blocks, 5 rows at 2 and 8 rows at 1); the two-pass form
// beyond. The kernel's shared-memory attribute and
// occupancy are set up on the handle's first launch (the configuration fixes both).
template <bool F32, int V>
inline int launch_ln_merge_pipe(vlproj_handle* h, const void* features, const ViewDesc* views, int n_views, int M,
                                float eps, __nv_bfloat16* A, cudaStream_t s) {
    const vlproj_config& c = h->cfg;
    const int64_t items = static_cast<int64_t>(M) * c.k * c.k;
    const size_t row_bytes = static_cast<size_t>(c.C) * (F32 ? 4 : 2);
    const int stages = static_cast<int>(std::min<size_t>(vlp::LNP_MAX_STAGES,
                                                         std::max<size_t>(2, (9u << 10) / row_bytes)));
    const size_t smem = vlp::LNP_BAR_BYTES + (c.has_ln ? 8 * static_cast<size_t>(c.C) : 0) +
                        static_cast<size_t>(vlp::LNP_WARPS) * stages * row_bytes;
    auto kern = vlp::vlp_ln_merge_pipe_kernel<F32, V>;
    if (h->lnp_per_sm == 0) {
        VLP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
        VLP_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&h->lnp_per_sm, kern, vlp::LNP_WARPS * 32, smem));
        h->lnp_per_sm = std::max(h->lnp_per_sm, 1);
    }
    const int64_t want = (items + vlp::LNP_WARPS - 1) / vlp::LNP_WARPS;
    const unsigned blocks =
        static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(h->num_sms) * h->lnp_per_sm)));
    kern<<<blocks, vlp::LNP_WARPS * 32, smem, s>>>(features, views, n_views, M, c.k, c.C, h->gamma, h->beta, eps,
                                                  c.has_ln, A, stages, h->wait_ns, h->status);
    VLP_CUDA(cudaGetLastError());
    return VLPROJ_OK;
}

// Source rows come from the view table `views` (n_views entries, on the device).
inline int launch_ln_merge(vlproj_handle* h, const void* features, const ViewDesc* views, int n_views, int M,
                           float eps, __nv_bfloat16* A, cudaStream_t s) {
    const vlproj_config& c = h->cfg;
    const int64_t items = static_cast<int64_t>(M) * c.k * c.k;
    if (items == 0) return VLPROJ_OK;
    const int nvec = c.C / 8;
    const bool f32 = c.feat_dtype == VLPROJ_FEAT_F32;
    if (nvec <= 64) return f32 ? launch_ln_merge_pipe<true, 2>(h, features, views, n_views, M, eps, A, s)
                               : launch_ln_merge_pipe<false, 2>(h, features, views, n_views, M, eps, A, s);
    if (nvec <= 160) return f32 ? launch_ln_merge_pipe<true, 5>(h, features, views, n_views, M, eps, A, s)
                                : launch_ln_merge_pipe<false, 5>(h, features, views, n_views, M, eps, A, s);
    if (nvec <= 256) return f32 ? launch_ln_merge_pipe<true, 8>(h, features, views, n_views, M, eps, A, s)
                                : launch_ln_merge_pipe<false, 8>(h, features, views, n_views, M, eps, A, s);
    const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
    if (f32)
        vlp::vlp_ln_merge_kernel<true><<<blocks, 256, 0, s>>>(features, views, n_views, M, c.k, c.C, h->gamma,
                                                              h->beta, eps, c.has_ln, A);
    else
        vlp::vlp_ln_merge_kernel<false><<<blocks, 256, 0, s>>>(features, views, n_views, M, c.k, c.C, h->gamma,
                                                               h->beta, eps, c.has_ln, A);
    VLP_CUDA(cudaGetLastError());
    return VLPROJ_OK;
}

inline int upload_plan(vlproj_handle* h, const Plan& pl, cudaStream_t s) {
    if (h->dviews.ptr == nullptr || h->dviews.cap < pl.views.size()) h->up_views.invalidate();
    if (h->dimages.ptr == nullptr || h->dimages.cap < pl.images.size()) h->up_images.invalidate();
    if (h->dviews.ensure(std::max<size_t>(pl.views.size(), 1))) return VLPROJ_ERR_CUDA;
    if (h->dimages.ensure(std::max<size_t>(pl.images.size(), 1))) return VLPROJ_ERR_CUDA;
    int rc = h->up_views.put(h->dviews.ptr, pl.views.data(), pl.views.size() * sizeof(ViewDesc), s);
    if (rc) return rc;
    return h->up_images.put(h->dimages.ptr, pl.images.data(), pl.images.size() * sizeof(ImageDesc), s);
}

// Defined in vlproj.cu: the forward's geometry + LayerNorm/convert + GEMM1 steps, and
// its middle layers (depth > 2).
int run_merge_gemm1(vlproj_handle* h, const Plan& pl, const void* features, const int32_t* pos, int dest_mode,
                    __nv_bfloat16* hidden, int64_t hidden_rows, cudaStream_t s, const vlp::ViewDesc* dviews);
int run_middle_layers(vlproj_handle* h, const Plan& pl, cudaStream_t s, const __nv_bfloat16** hlast);

}  // namespace vlp_host
