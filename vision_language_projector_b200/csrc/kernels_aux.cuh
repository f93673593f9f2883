// Memory-bound kernels around the projector GEMMs (sm_100a):
//   placeholder index   - compact the flat positions holding the image id, in
//                         order, and check their count against the closed form;
//   geometry            - per merged token: where its k x k neighbourhood starts
//                         in the packed features, which neighbours lie inside the
//                         grid, and which embedding row its projection goes to;
//   LayerNorm           - pre-merge LayerNorm per patch (and fp32 -> bf16), bf16 out,
//                         either in patch order or already merged (GEMM1's A operand);
//   special rows        - copy the learned newline / view-separator vectors into
//                         their placeholder rows (2D tiling);
//   W1 permutation      - reorder W1's input columns from c*k*k + p to p*C + c.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace vlp {

constexpr int ERR_TOKEN_COUNT = -4;

// ---------------------------------------------------------------- placeholder index
constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ITEMS = 16;
constexpr int SCAN_CHUNK = SCAN_THREADS * SCAN_ITEMS;     // ids per block

__device__ __forceinline__ int block_sum_256(int v, int* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < SCAN_THREADS / 32; ++w) t += red[w];
    return t;
}

// counts[b] = number of placeholders in ids[b*SCAN_CHUNK, (b+1)*SCAN_CHUNK)
static __global__ void __launch_bounds__(SCAN_THREADS) vlp_count_kernel(const int64_t* __restrict__ ids, int64_t n,
                                                                 int64_t token, int32_t* __restrict__ counts) {
    __shared__ int red[SCAN_THREADS / 32];
    const int64_t start = static_cast<int64_t>(blockIdx.x) * SCAN_CHUNK;
    int c = 0;
#pragma unroll
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        const int64_t idx = start + i * SCAN_THREADS + threadIdx.x;
        if (idx < n && __ldg(&ids[idx]) == token) ++c;
    }
    c = block_sum_256(c, red);
    if (threadIdx.x == 0) counts[blockIdx.x] = c;
}

// Writes pos[j] = flat index of the j-th placeholder (j < R), in order. Each block
// finds its starting rank from the counts of the blocks before it, then ranks its
// own placeholders with warp ballots. Block 0 records whether the total equals R.
static __global__ void __launch_bounds__(SCAN_THREADS) vlp_compact_kernel(const int64_t* __restrict__ ids, int64_t n,
                                                                   int64_t token, const int32_t* __restrict__ counts,
                                                                   int nblocks, int32_t* __restrict__ pos, int64_t R,
                                                                   int* fwd_status, int* err) {
    __shared__ int red[SCAN_THREADS / 32];
    __shared__ int warp_cnt[SCAN_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int pre = 0, tot = 0;
    for (int b = threadIdx.x; b < nblocks; b += SCAN_THREADS) {
        const int c = counts[b];
        tot += c;
        if (b < static_cast<int>(blockIdx.x)) pre += c;
    }
    pre = block_sum_256(pre, red);
    tot = block_sum_256(tot, red);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const int st = (static_cast<int64_t>(tot) == R) ? 0 : ERR_TOKEN_COUNT;
        *fwd_status = st;
        if (st != 0) atomicCAS(err, 0, st);
    }
    const int64_t start = static_cast<int64_t>(blockIdx.x) * SCAN_CHUNK;
    int64_t run = pre;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        const int64_t idx = start + i * SCAN_THREADS + threadIdx.x;
        const bool flag = idx < n && __ldg(&ids[idx]) == token;
        const unsigned bal = __ballot_sync(0xffffffffu, flag);
        if (lane == 0) warp_cnt[warp] = __popc(bal);
        __syncthreads();
        int before = 0, all = 0;
#pragma unroll
        for (int w = 0; w < SCAN_THREADS / 32; ++w) {
            const int c = warp_cnt[w];
            before += (w < warp) ? c : 0;
            all += c;
        }
        const int64_t rank = run + before + __popc(bal & lt_mask);
        if (flag && rank < R) pos[rank] = static_cast<int32_t>(idx);
        run += all;
        __syncthreads();
    }
}

// ---------------------------------------------------------------- geometry
struct ViewDesc {
    int64_t patch_start;   // first patch row of the view in the packed features
    int32_t tok_start;     // first GEMM row of the view (runs padded to the im2col chunk when varlen)
    int32_t tok_real;      // merged tokens of all earlier views (no padding)
    int32_t h, w;          // patch grid
    int32_t hp, wp;        // merged grid: ceil(h/k), ceil(w/k)
    int32_t row_base;      // first assembled row of the view's image (over all images)
    int32_t view_in_image; // 0 = global view (or the only view), t+1 = local tile t
    int32_t tw, th;        // image tiling (0 when untiled)
    int32_t tail;          // 2D tiling with the global view after the local tiles
};

// Assembled row (inside the image) of merged token (i, j) of a view.
__device__ __forceinline__ int64_t assembled_row(const ViewDesc& V, int i, int j) {
    if (V.tw == 0) return static_cast<int64_t>(i) * V.wp + j;
    const int64_t global_rows = static_cast<int64_t>(V.hp) * (V.wp + 1);
    const int64_t local_cols = static_cast<int64_t>(V.tw) * V.wp + 1;
    const int64_t local_rows = static_cast<int64_t>(V.th) * V.hp * local_cols;
    const int64_t g0 = V.tail ? local_rows + 1 : 0;           // first row of the global block
    const int64_t l0 = V.tail ? 0 : global_rows + 1;          // first row of the local block
    if (V.view_in_image == 0) return g0 + static_cast<int64_t>(i) * (V.wp + 1) + j;
    const int t = V.view_in_image - 1, ty = t / V.tw, tx = t - ty * V.tw;
    return l0 + (static_cast<int64_t>(ty) * V.hp + i) * local_cols + static_cast<int64_t>(tx) * V.wp + j;
}

__device__ __forceinline__ int find_view(const ViewDesc* views, int n_views, int m) {
    int lo = 0, hi = n_views - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (views[mid].tok_start <= m) lo = mid; else hi = mid - 1;
    }
    return lo;
}

constexpr int DEST_NONE = 0;      // no destination table
constexpr int DEST_EMBED = 1;     // rowdest[m] = embedding row of the placeholder that takes token m
constexpr int DEST_COMPACT = 2;   // rowdest[m] = merged-token index (views in order, no padding)
constexpr int DEST_ROW = 3;       // rowdest[m] = assembled row of token m (the rows of the batch in order)

// One thread per GEMM row m (and per im2col chunk): gather metadata for the cp.async
// path, the destination of the row, and the im2col coordinates of each chunk's
// first token. Rows in a view's padding get no destination and zero gather masks.
static __global__ void __launch_bounds__(256) vlp_geometry_kernel(const ViewDesc* __restrict__ views, int n_views, int M,
                                                           int k, const int32_t* __restrict__ pos, int64_t R,
                                                           int dest_mode, int2* __restrict__ gmeta,
                                                           int32_t* __restrict__ rowdest, int4* __restrict__ chunks,
                                                           int n_chunks, int chunk, int uniform) {
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m < n_chunks) {
        const int first = m * chunk;
        int4 e;
        if (first >= M) {
            // past the last GEMM row: any in-range start will do, these rows are never stored
            e = make_int4(0, 0, 0, 0);
        } else {
            const int v = find_view(views, n_views, first);
            const ViewDesc& V = views[v];
            const int t = first - V.tok_start;
            const int i = t / V.wp, j = t - (t / V.wp) * V.wp;
            e = uniform ? make_int4(0, k * j, k * i, v) : make_int4(v, k * j, k * i, 0);
        }
        if (chunks != nullptr) chunks[m] = e;
    }
    if (m >= M) return;
    const ViewDesc V = views[find_view(views, n_views, m)];
    const int t = m - V.tok_start;
    const bool real = t < V.hp * V.wp;
    const int i = real ? t / V.wp : 0, j = real ? t - i * V.wp : 0;
    if (gmeta != nullptr) {
        const int64_t base = V.patch_start + static_cast<int64_t>(k * i) * V.w + k * j;
        uint32_t mask = 0;
        if (real)
            for (int dy = 0; dy < k; ++dy)
                for (int dx = 0; dx < k; ++dx)
                    if (k * i + dy < V.h && k * j + dx < V.w) mask |= 1u << (dy * k + dx);
        gmeta[m] = make_int2(static_cast<int>(base), static_cast<int>((static_cast<uint32_t>(V.w) << 16) | mask));
    }
    if (dest_mode == DEST_EMBED) {
        const int64_t g = V.row_base + assembled_row(V, i, j);
        rowdest[m] = (real && g >= 0 && g < R) ? pos[g] : -1;
    } else if (dest_mode == DEST_COMPACT) {
        rowdest[m] = real ? V.tok_real + t : -1;
    } else if (dest_mode == DEST_ROW) {
        const int64_t g = V.row_base + assembled_row(V, i, j);
        rowdest[m] = (real && g >= 0 && g < R) ? static_cast<int32_t>(g) : -1;
    }
}

// ---------------------------------------------------------------- LayerNorm / convert
// One warp per patch row: y = bf16(((x - mean) * rstd) * gamma + beta) (biased
// variance, fp32 statistics) or, without LayerNorm, y = bf16(x). C % 8 == 0.
template <bool kF32In>
static __global__ void __launch_bounds__(256) vlp_layernorm_kernel(const void* __restrict__ x, int64_t P, int C,
                                                            const float* __restrict__ gamma,
                                                            const float* __restrict__ beta, float eps, int has_ln,
                                                            __nv_bfloat16* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= P) return;
    const int nvec = C / 8;
    auto load8 = [&](int v, float (&f)[8]) {
        if (kF32In) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * C) + 2 * v;
            const float4 a = __ldg(src), b = __ldg(src + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        } else {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + row * C) + v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                f[2 * e] = __uint_as_float(w[e] << 16);
                f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    };
    float mean = 0.f, rstd = 1.f;
    if (has_ln) {
        float s = 0.f;
        for (int v = lane; v < nvec; v += 32) {
            float f[8];
            load8(v, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) s += f[e];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        mean = s / static_cast<float>(C);
        float q = 0.f;
        for (int v = lane; v < nvec; v += 32) {
            float f[8];
            load8(v, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float d = f[e] - mean;
                q += d * d;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        rstd = rsqrtf(q / static_cast<float>(C) + eps);
    }
    for (int v = lane; v < nvec; v += 32) {
        float f[8];
        load8(v, f);
        if (has_ln) {
            const float4* g4 = reinterpret_cast<const float4*>(gamma) + 2 * v;
            const float4* b4 = reinterpret_cast<const float4*>(beta) + 2 * v;
            const float4 g0 = __ldg(g4), g1 = __ldg(g4 + 1), b0 = __ldg(b4), b1 = __ldg(b4 + 1);
            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (f[e] - mean) * rstd * gg[e] + bb[e];
        }
        uint4 o;
        __nv_bfloat162 t0 = __floats2bfloat162_rn(f[0], f[1]), t1 = __floats2bfloat162_rn(f[2], f[3]);
        __nv_bfloat162 t2 = __floats2bfloat162_rn(f[4], f[5]), t3 = __floats2bfloat162_rn(f[6], f[7]);
        o.x = *reinterpret_cast<uint32_t*>(&t0);
        o.y = *reinterpret_cast<uint32_t*>(&t1);
        o.z = *reinterpret_cast<uint32_t*>(&t2);
        o.w = *reinterpret_cast<uint32_t*>(&t3);
        reinterpret_cast<uint4*>(y + row * C)[v] = o;
    }
}

// ---------------------------------------------------------------- LayerNorm + merge
// One warp per (merged token m, position p = dy*k + dx): the patch at (k*i+dy, k*j+dx)
// of m's view (from gmeta), LayerNorm'd (when has_ln) and rounded to bf16, lands at
// A[m][p*C : (p+1)*C]; positions in the high-end pad are written as zeros. Each
// patch is read once, and A is GEMM1's operand in the kernel's K order. The
// statistics and rounding are those of vlp_layernorm_kernel, so A holds exactly the
// values the gathering paths read from its output.
template <bool kF32In>
static __global__ void __launch_bounds__(256) vlp_ln_merge_kernel(const void* __restrict__ x, const int2* __restrict__ gmeta,
                                                           int M, int k, int C, const float* __restrict__ gamma,
                                                           const float* __restrict__ beta, float eps, int has_ln,
                                                           __nv_bfloat16* __restrict__ A) {
    const int lane = threadIdx.x & 31;
    const int kk = k * k;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(M) * kk) return;
    const int m = static_cast<int>(item / kk), p = static_cast<int>(item - static_cast<int64_t>(m) * kk);
    const int dy = p / k, dx = p - dy * k;
    const int2 g = gmeta[m];
    const uint32_t wm = static_cast<uint32_t>(g.y);
    const int nvec = C / 8;
    uint4* dst = reinterpret_cast<uint4*>(A + (static_cast<int64_t>(m) * kk + p) * C);
    if (!((wm >> p) & 1u)) {
        for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        return;
    }
    const int64_t row = static_cast<int64_t>(g.x) + dy * static_cast<int>(wm >> 16) + dx;
    auto load8 = [&](int v, float (&f)[8]) {
        if (kF32In) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * C) + 2 * v;
            const float4 a = __ldg(src), b = __ldg(src + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        } else {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + row * C) + v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                f[2 * e] = __uint_as_float(w[e] << 16);
                f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    };
    float mean = 0.f, rstd = 1.f;
    if (has_ln) {
        float s = 0.f;
        for (int v = lane; v < nvec; v += 32) {
            float f[8];
            load8(v, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) s += f[e];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        mean = s / static_cast<float>(C);
        float q = 0.f;
        for (int v = lane; v < nvec; v += 32) {
            float f[8];
            load8(v, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float d = f[e] - mean;
                q += d * d;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        rstd = rsqrtf(q / static_cast<float>(C) + eps);
    }
    for (int v = lane; v < nvec; v += 32) {
        float f[8];
        load8(v, f);
        if (has_ln) {
            const float4* g4 = reinterpret_cast<const float4*>(gamma) + 2 * v;
            const float4* b4 = reinterpret_cast<const float4*>(beta) + 2 * v;
            const float4 g0 = __ldg(g4), g1 = __ldg(g4 + 1), b0 = __ldg(b4), b1 = __ldg(b4 + 1);
            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (f[e] - mean) * rstd * gg[e] + bb[e];
        }
        uint4 o;
        __nv_bfloat162 t0 = __floats2bfloat162_rn(f[0], f[1]), t1 = __floats2bfloat162_rn(f[2], f[3]);
        __nv_bfloat162 t2 = __floats2bfloat162_rn(f[4], f[5]), t3 = __floats2bfloat162_rn(f[6], f[7]);
        o.x = *reinterpret_cast<uint32_t*>(&t0);
        o.y = *reinterpret_cast<uint32_t*>(&t1);
        o.z = *reinterpret_cast<uint32_t*>(&t2);
        o.w = *reinterpret_cast<uint32_t*>(&t3);
        dst[v] = o;
    }
}

// Single-pass form of vlp_ln_merge_kernel for C <= 256 * kVec: each lane keeps its
// kVec 8-channel vectors of the patch in registers, so the patch is read from memory
// once. Same statistics (sum, then sum of squared deviations, in fp32) and rounding.
template <bool kF32In, int kVec>
static __global__ void __launch_bounds__(256) vlp_ln_merge_regs_kernel(const void* __restrict__ x,
                                                                const int2* __restrict__ gmeta, int M, int k, int C,
                                                                const float* __restrict__ gamma,
                                                                const float* __restrict__ beta, float eps, int has_ln,
                                                                __nv_bfloat16* __restrict__ A) {
    const int lane = threadIdx.x & 31;
    const int kk = k * k;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(M) * kk) return;
    const int m = static_cast<int>(item / kk), p = static_cast<int>(item - static_cast<int64_t>(m) * kk);
    const int dy = p / k, dx = p - dy * k;
    const int2 g = gmeta[m];
    const uint32_t wm = static_cast<uint32_t>(g.y);
    const int nvec = C / 8;
    uint4* dst = reinterpret_cast<uint4*>(A + (static_cast<int64_t>(m) * kk + p) * C);
    if (!((wm >> p) & 1u)) {
        for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        return;
    }
    const int64_t row = static_cast<int64_t>(g.x) + dy * static_cast<int>(wm >> 16) + dx;
    float f[kVec][8];
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) {
            if (kF32In) {
                const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * C) + 2 * v;
                const float4 a = __ldg(src), b = __ldg(src + 1);
                f[i][0] = a.x; f[i][1] = a.y; f[i][2] = a.z; f[i][3] = a.w;
                f[i][4] = b.x; f[i][5] = b.y; f[i][6] = b.z; f[i][7] = b.w;
            } else {
                const uint4 u =
                    __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + row * C) + v);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    f[i][2 * e] = __uint_as_float(w[e] << 16);
                    f[i][2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[i][e] = 0.f;
        }
    }
    float mean = 0.f, rstd = 1.f;
    if (has_ln) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) s += f[i][e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        mean = s / static_cast<float>(C);
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            if (lane + 32 * i < nvec) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float d = f[i][e] - mean;
                    q += d * d;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        rstd = rsqrtf(q / static_cast<float>(C) + eps);
    }
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
        const int v = lane + 32 * i;
        if (v >= nvec) continue;
        if (has_ln) {
            const float4* g4 = reinterpret_cast<const float4*>(gamma) + 2 * v;
            const float4* b4 = reinterpret_cast<const float4*>(beta) + 2 * v;
            const float4 g0 = __ldg(g4), g1 = __ldg(g4 + 1), b0 = __ldg(b4), b1 = __ldg(b4 + 1);
            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) f[i][e] = (f[i][e] - mean) * rstd * gg[e] + bb[e];
        }
        uint4 o;
        __nv_bfloat162 t0 = __floats2bfloat162_rn(f[i][0], f[i][1]), t1 = __floats2bfloat162_rn(f[i][2], f[i][3]);
        __nv_bfloat162 t2 = __floats2bfloat162_rn(f[i][4], f[i][5]), t3 = __floats2bfloat162_rn(f[i][6], f[i][7]);
        o.x = *reinterpret_cast<uint32_t*>(&t0);
        o.y = *reinterpret_cast<uint32_t*>(&t1);
        o.z = *reinterpret_cast<uint32_t*>(&t2);
        o.w = *reinterpret_cast<uint32_t*>(&t3);
        dst[v] = o;
    }
}

// ---------------------------------------------------------------- newline / separator rows
struct ImageDesc {
    int32_t row_base;       // first assembled row of the image (over all images)
    int32_t hp, wp, tw, th; // merged grid and tiling
    int32_t tail;           // global view after the local tiles
};

// Row, inside its image, of special row n of a 2D-tiled image:
//   n <  hp            newline closing global row n
//   n <  hp + th*hp    newline closing local canvas row n - hp
//   n == hp + th*hp    the view separator
__device__ __forceinline__ int64_t special_row(const ImageDesc& I, int n) {
    const int n_nl = I.hp + I.th * I.hp;
    const int64_t global_rows = static_cast<int64_t>(I.hp) * (I.wp + 1);
    const int64_t local_cols = static_cast<int64_t>(I.tw) * I.wp + 1;
    const int64_t local_rows = static_cast<int64_t>(I.th) * I.hp * local_cols;
    const int64_t g0 = I.tail ? local_rows + 1 : 0;
    const int64_t l0 = I.tail ? 0 : global_rows + 1;
    if (n < I.hp) return g0 + static_cast<int64_t>(n) * (I.wp + 1) + I.wp;
    if (n < n_nl) return l0 + static_cast<int64_t>(n - I.hp) * local_cols + local_cols - 1;
    return I.tail ? local_rows : global_rows;
}

// blockIdx.y = image, blockIdx.x = special row n of that image (see special_row). The row
// goes to out[pos[g]] for assembled row g, or to out[g] when pos is null (rows in
// assembled order); fwd_status null = no count check.
static __global__ void __launch_bounds__(128) vlp_special_rows_kernel(const ImageDesc* __restrict__ imgs,
                                                               const int32_t* __restrict__ pos, int64_t R,
                                                               const __nv_bfloat16* __restrict__ newline,
                                                               const __nv_bfloat16* __restrict__ sep,
                                                               __nv_bfloat16* __restrict__ out, int64_t out_rows,
                                                               int N, const int* __restrict__ fwd_status) {
    if (fwd_status != nullptr && *fwd_status != 0) return;
    const ImageDesc I = imgs[blockIdx.y];
    const int n = blockIdx.x;
    const int n_nl = I.hp + I.th * I.hp;
    if (n > n_nl) return;
    const __nv_bfloat16* src = n < n_nl ? newline : sep;
    const int64_t g = I.row_base + special_row(I, n);
    if (g < 0 || g >= R) return;
    const int64_t d = pos != nullptr ? pos[g] : g;
    if (d < 0 || d >= out_rows) return;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(out + d * N);
    for (int v = threadIdx.x; v < N / 8; v += blockDim.x) d4[v] = __ldg(&s4[v]);
}

// ---------------------------------------------------------------- token-embedding lookup
// One warp per row: out[r] = table[ids[r]] for every id that is not the placeholder; an
// id outside [0, vocab) writes a zero row and latches VLPROJ_ERR_INVALID_ARG.
static __global__ void __launch_bounds__(256) vlp_embed_lookup_kernel(const int64_t* __restrict__ ids, int64_t n,
                                                               int64_t token, const __nv_bfloat16* __restrict__ table,
                                                               int64_t vocab, __nv_bfloat16* __restrict__ out, int N,
                                                               int* err) {
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (r >= n) return;
    const int64_t id = __ldg(&ids[r]);
    if (id == token) return;
    uint4* d4 = reinterpret_cast<uint4*>(out + r * N);
    const int nvec = N / 8;
    if (id < 0 || id >= vocab) {
        for (int v = lane; v < nvec; v += 32) d4[v] = make_uint4(0, 0, 0, 0);
        if (lane == 0) atomicCAS(err, 0, -1);
        return;
    }
    const uint4* s4 = reinterpret_cast<const uint4*>(table + id * N);
    for (int v = lane; v < nvec; v += 32) d4[v] = __ldg(&s4[v]);
}

// rows_out[j] = out[pos[j]] for the R assembled rows (nothing when the count check failed).
static __global__ void __launch_bounds__(256) vlp_gather_rows_kernel(const int32_t* __restrict__ pos, int64_t R,
                                                              const __nv_bfloat16* __restrict__ out, int64_t out_rows,
                                                              int N, __nv_bfloat16* __restrict__ rows_out,
                                                              const int* __restrict__ fwd_status) {
    if (*fwd_status != 0) return;
    const int lane = threadIdx.x & 31;
    const int64_t j = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (j >= R) return;
    const int64_t d = pos[j];
    if (d < 0 || d >= out_rows) return;
    const uint4* s4 = reinterpret_cast<const uint4*>(out + d * N);
    uint4* d4 = reinterpret_cast<uint4*>(rows_out + j * N);
    for (int v = lane; v < N / 8; v += 32) d4[v] = s4[v];
}

// ---------------------------------------------------------------- W1 column permutation
// dst[n][p*C + c] = src[n][c*kk + p] for p < kk = k*k (channel-outermost input);
// with position_outer the columns are copied unchanged.
static __global__ void vlp_permute_w1_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                      int64_t N1, int C, int kk, int position_outer) {
    const int64_t K1 = static_cast<int64_t>(C) * kk;
    const int64_t total = N1 * K1;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t n = e / K1, q = e - n * K1;     // q = p*C + c in the destination
        const int64_t p = q / C, c = q - p * C;
        const int64_t s = position_outer ? q : c * kk + p;
        dst[e] = src[n * K1 + s];
    }
}

}  // namespace vlp
