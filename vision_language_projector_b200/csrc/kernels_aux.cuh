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

#include "ptx.cuh"

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

// One block of SCAN_TOTAL_THREADS turns the per-block counts into exclusive prefix sums
// in place and appends the total: counts[b] <- counts[0] + ... + counts[b-1] for b <
// nblocks, counts[nblocks] <- the sum of all (counts holds nblocks + 1 entries). Thread t
// owns the contiguous segment [t*seg, (t+1)*seg) with seg = ceil(nblocks / threads); the
// segment sums are scanned across the block (warp shuffles, then the warp totals), so the
// work is O(nblocks) however many blocks there are. The sum is below 2^31 (n < 2^31).
constexpr int SCAN_TOTAL_THREADS = 1024;
static __global__ void __launch_bounds__(SCAN_TOTAL_THREADS) vlp_scan_counts_kernel(int32_t* __restrict__ counts,
                                                                                     int nblocks) {
    __shared__ int warp_tot[SCAN_TOTAL_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = (nblocks + SCAN_TOTAL_THREADS - 1) / SCAN_TOTAL_THREADS;
    const int b0 = min(nblocks, static_cast<int>(threadIdx.x) * seg), b1 = min(nblocks, b0 + seg);
    int own = 0;
    for (int b = b0; b < b1; ++b) own += counts[b];
    // inclusive scan of the segment sums inside the warp
    int inc = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < SCAN_TOTAL_THREADS / 32; ++w) {
        const int t = warp_tot[w];
        before += (w < warp) ? t : 0;
        total += t;
    }
    int run = before + inc - own;          // exclusive prefix of this thread's segment
    for (int b = b0; b < b1; ++b) {
        const int c = counts[b];
        counts[b] = run;
        run += c;
    }
    if (threadIdx.x == 0) counts[nblocks] = total;
}

// Writes pos[j] = flat index of the j-th placeholder (j < R), in order. `prefix` holds
// the exclusive prefix sums of the per-block counts and their total at prefix[nblocks]
// (vlp_scan_counts_kernel; with nblocks == 0 only prefix[0] = 0 is read). Each block
// starts at its own prefix and ranks its placeholders with warp ballots. Block 0 writes
// the total to *count_out (when given) and, when fwd_status is given, whether the total
// equals R (latching VLPROJ_ERR_TOKEN_COUNT in *err when it does not).
static __global__ void __launch_bounds__(SCAN_THREADS) vlp_compact_kernel(const int64_t* __restrict__ ids, int64_t n,
                                                                   int64_t token, const int32_t* __restrict__ prefix,
                                                                   int nblocks, int32_t* __restrict__ pos, int64_t R,
                                                                   int* fwd_status, int* err, int64_t* count_out) {
    __shared__ int warp_cnt[SCAN_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int pre = nblocks > 0 ? prefix[blockIdx.x] : 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const int tot = nblocks > 0 ? prefix[nblocks] : 0;
        if (count_out != nullptr) *count_out = tot;
        if (fwd_status != nullptr) {
            const int st = (static_cast<int64_t>(tot) == R) ? 0 : ERR_TOKEN_COUNT;
            *fwd_status = st;
            if (st != 0 && err != nullptr) atomicCAS(err, 0, st);
        }
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

// Blocks of SCAN_CHUNK ids the index step uses for n ids; its count buffer holds one
// more entry than that (the total).
inline int scan_blocks(int64_t n) { return static_cast<int>((n + SCAN_CHUNK - 1) / SCAN_CHUNK); }

// The whole placeholder-index step on `s`: count per block, prefix sums, compact.
// `counts` holds scan_blocks(n) + 1 entries; pos, R, fwd_status, err, count_out as in
// vlp_compact_kernel. Adds the number of kernels launched to *launches. n < 2^31.
inline cudaError_t enqueue_placeholder_index(const int64_t* ids, int64_t n, int64_t token, int32_t* counts,
                                             int32_t* pos, int64_t R, int* fwd_status, int* err, int64_t* count_out,
                                             cudaStream_t s, int64_t* launches) {
    const int nblocks = scan_blocks(n);
    if (nblocks > 0) {
        vlp_count_kernel<<<nblocks, SCAN_THREADS, 0, s>>>(ids, n, token, counts);
        vlp_scan_counts_kernel<<<1, SCAN_TOTAL_THREADS, 0, s>>>(counts, nblocks);
        *launches += 2;
    }
    vlp_compact_kernel<<<nblocks > 0 ? nblocks : 1, SCAN_THREADS, 0, s>>>(ids, n, token, counts, nblocks, pos, R,
                                                                         fwd_status, err, count_out);
    *launches += 1;
    return cudaGetLastError();
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
// y = bf16(((x - mean) * rstd) * gamma + beta) per patch row, biased variance, fp32
// statistics, or y = bf16(x) without a LayerNorm; C % 8 == 0. One warp per row; lane l
// owns the 8-channel vectors v = l, l + 32, ... and works on channel pairs (2e, 2e+1)
// held as packed fp32x2, two channels per add / mul / fma instruction.
//
// Every kernel below reduces in the same order, so they produce the same bits: a
// lane accumulates its vectors in increasing v into an (even, odd) pair of sums,
// adds the pair, and the warp combines lanes by an xor tree; the sum of squared
// deviations from the mean likewise.

// The 8 channels of vector v of a row as 4 packed pairs.
template <bool kF32In>
__device__ __forceinline__ void ln_load_pairs(const void* __restrict__ x, int64_t row, int C, int v,
                                              uint64_t (&q)[4]) {
    if (kF32In) {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * C) + 2 * v;
        const float4 a = __ldg(src), b = __ldg(src + 1);
        q[0] = f2_pack(a.x, a.y);
        q[1] = f2_pack(a.z, a.w);
        q[2] = f2_pack(b.x, b.y);
        q[3] = f2_pack(b.z, b.w);
    } else {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + row * C) + v);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) q[e] = f2_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
    }
}

// Same from a row staged in shared memory.
template <bool kF32In>
__device__ __forceinline__ void ln_smem_pairs(const uint8_t* st, int v, uint64_t (&q)[4]) {
    if (kF32In) {
        const float4 a = reinterpret_cast<const float4*>(st)[2 * v];
        const float4 b = reinterpret_cast<const float4*>(st)[2 * v + 1];
        q[0] = f2_pack(a.x, a.y);
        q[1] = f2_pack(a.z, a.w);
        q[2] = f2_pack(b.x, b.y);
        q[3] = f2_pack(b.z, b.w);
    } else {
        const uint4 u = reinterpret_cast<const uint4*>(st)[v];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) q[e] = f2_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
    }
}

// Sum of the pair accumulator's halves, then across the warp.
__device__ __forceinline__ float ln_warp_total(uint64_t acc) {
    float a, b;
    f2_unpack(acc, a, b);
    float t = a + b;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return t;
}

// bf16 of 8 channels: d = x - mean (packed), y = (d * rstd) * gamma + beta, with
// gamma / beta of the 8 channels in g0, g1 / b0, b1.
__device__ __forceinline__ uint4 ln_out_pairs(const uint64_t (&d)[4], uint64_t rstd2, float4 g0, float4 g1, float4 b0,
                                              float4 b1) {
    const uint64_t gg[4] = {f2_pack(g0.x, g0.y), f2_pack(g0.z, g0.w), f2_pack(g1.x, g1.y), f2_pack(g1.z, g1.w)};
    const uint64_t bb[4] = {f2_pack(b0.x, b0.y), f2_pack(b0.z, b0.w), f2_pack(b1.x, b1.y), f2_pack(b1.z, b1.w)};
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float lo, hi;
        f2_unpack(f2_fma(f2_mul(d[e], rstd2), gg[e], bb[e]), lo, hi);
        __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
        w[e] = *reinterpret_cast<uint32_t*>(&t);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// bf16 of 8 channels without a LayerNorm.
__device__ __forceinline__ uint4 ln_convert_pairs(const uint64_t (&x)[4]) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float lo, hi;
        f2_unpack(x[e], lo, hi);
        __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
        w[e] = *reinterpret_cast<uint32_t*>(&t);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Statistics of the row `row` read vector by vector from memory: mean, 1/sqrt(var + eps).
template <bool kF32In>
__device__ __forceinline__ void ln_row_stats(const void* __restrict__ x, int64_t row, int C, int lane, float eps,
                                             float& mean, float& rstd) {
    const int nvec = C / 8;
    uint64_t acc = 0;
    for (int v = lane; v < nvec; v += 32) {
        uint64_t q[4];
        ln_load_pairs<kF32In>(x, row, C, v, q);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc = f2_add(acc, q[e]);
    }
    const float inv_c = 1.0f / static_cast<float>(C);
    mean = ln_warp_total(acc) * inv_c;
    const uint64_t nm = f2_splat(-mean);
    acc = 0;
    for (int v = lane; v < nvec; v += 32) {
        uint64_t q[4];
        ln_load_pairs<kF32In>(x, row, C, v, q);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint64_t d = f2_add(q[e], nm);
            acc = f2_fma(d, d, acc);
        }
    }
    rstd = rsqrtf(ln_warp_total(acc) * inv_c + eps);
}

// Normalise row `row` of x into dst (bf16, C channels), re-reading x vector by vector.
template <bool kF32In>
__device__ __forceinline__ void ln_row_write(const void* __restrict__ x, int64_t row, int C, int lane,
                                             const float* __restrict__ gamma, const float* __restrict__ beta,
                                             float eps, int has_ln, uint4* __restrict__ dst) {
    const int nvec = C / 8;
    float mean = 0.f, rstd = 1.f;
    if (has_ln) ln_row_stats<kF32In>(x, row, C, lane, eps, mean, rstd);
    const uint64_t nm = f2_splat(-mean), r2 = f2_splat(rstd);
    for (int v = lane; v < nvec; v += 32) {
        uint64_t q[4];
        ln_load_pairs<kF32In>(x, row, C, v, q);
        if (has_ln) {
#pragma unroll
            for (int e = 0; e < 4; ++e) q[e] = f2_add(q[e], nm);
            const float4* g4 = reinterpret_cast<const float4*>(gamma) + 2 * v;
            const float4* b4 = reinterpret_cast<const float4*>(beta) + 2 * v;
            dst[v] = ln_out_pairs(q, r2, __ldg(g4), __ldg(g4 + 1), __ldg(b4), __ldg(b4 + 1));
        } else {
            dst[v] = ln_convert_pairs(q);
        }
    }
}

// Patch order: row p of the features -> row p of y.
template <bool kF32In>
static __global__ void __launch_bounds__(256) vlp_layernorm_kernel(const void* __restrict__ x, int64_t P, int C,
                                                            const float* __restrict__ gamma,
                                                            const float* __restrict__ beta, float eps, int has_ln,
                                                            __nv_bfloat16* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= P) return;
    ln_row_write<kF32In>(x, row, C, lane, gamma, beta, eps, has_ln, reinterpret_cast<uint4*>(y + row * C));
}

// ---------------------------------------------------------------- LayerNorm + merge
// Item (merged token m, position p = dy*k + dx): the patch at (k*i+dy, k*j+dx) of m's
// view (found in the view table), LayerNorm'd (when has_ln) and rounded to bf16, lands at
// A[m][p*C : (p+1)*C]; positions in the high-end pad are written as zeros. Each patch
// is read from memory once and A is GEMM1's operand in the kernel's K order. Values
// equal vlp_layernorm_kernel's output bit for bit, so A holds exactly what the
// gathering paths read.

// Source row of item (m, p), or -1 for a zero pad.
__device__ __forceinline__ int64_t merge_source_row(const int2* __restrict__ gmeta, int m, int p, int k) {
    const int2 g = __ldg(gmeta + m);
    const uint32_t wm = static_cast<uint32_t>(g.y);
    if (!((wm >> p) & 1u)) return -1;
    return static_cast<int64_t>(g.x) + (p / k) * static_cast<int>(wm >> 16) + (p % k);
}

// The same from the view table (no gather metadata needed): token m of its view is
// merged-grid cell (i, j), tap p = dy * k + dx is patch (k i + dy, k j + dx) if that lies
// inside the view's grid.
__device__ __forceinline__ int64_t merge_source_row(const ViewDesc* __restrict__ views, int n_views, int m, int p,
                                                    int k) {
    const ViewDesc& V = views[find_view(views, n_views, m)];
    const int t = m - V.tok_start;
    if (t >= V.hp * V.wp) return -1;
    const int i = t / V.wp, j = t - (t / V.wp) * V.wp;
    const int y = k * i + p / k, x = k * j + p % k;
    if (y >= V.h || x >= V.w) return -1;
    return V.patch_start + static_cast<int64_t>(y) * V.w + x;
}

// Any C: one warp per item, the row re-read from memory for each pass.
template <bool kF32In>
static __global__ void __launch_bounds__(256) vlp_ln_merge_kernel(const void* __restrict__ x,
                                                           const ViewDesc* __restrict__ views, int n_views,
                                                           int M, int k, int C, const float* __restrict__ gamma,
                                                           const float* __restrict__ beta, float eps, int has_ln,
                                                           __nv_bfloat16* __restrict__ A) {
    const int lane = threadIdx.x & 31;
    const int kk = k * k;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (item >= static_cast<int64_t>(M) * kk) return;
    const int m = static_cast<int>(item / kk), p = static_cast<int>(item - static_cast<int64_t>(m) * kk);
    uint4* dst = reinterpret_cast<uint4*>(A + item * C);
    const int64_t row = merge_source_row(views, n_views, m, p, k);
    if (row < 0) {
        for (int v = lane; v < C / 8; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        return;
    }
    ln_row_write<kF32In>(x, row, C, lane, gamma, beta, eps, has_ln, dst);
}

// LayerNorm statistics for the GEMM that normalises its A operand in shared memory
// (A_TGATHER_LN): for GEMM row m < rows and tap p < k*k, stats[p * rows + m] = (mean,
// rstd) of the patch at tap p of merged token m, computed by ln_row_stats (the same
// arithmetic, in the same order, as every LayerNorm kernel here, so the normalised values
// match theirs bit for bit), or (0, 0) where the tap lies in the high-end pad or m >= M.
// One warp per (p, m); consecutive warps take consecutive m at one tap. Every patch of the
// batch is read once (twice from the same warp: mean, then variance, the second from L1).
template <bool kF32In>
static __global__ void __launch_bounds__(256) vlp_ln_stats_kernel(const void* __restrict__ x,
                                                           const ViewDesc* __restrict__ views, int n_views, int M,
                                                           int64_t rows, int k, int C, float eps,
                                                           float2* __restrict__ stats) {
    const int lane = threadIdx.x & 31;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (item >= rows * k * k) return;
    const int p = static_cast<int>(item / rows);
    const int m = static_cast<int>(item - static_cast<int64_t>(p) * rows);
    const int64_t src = m < M ? merge_source_row(views, n_views, m, p, k) : -1;
    float mean = 0.f, rstd = 0.f;
    if (src >= 0) ln_row_stats<kF32In>(x, src, C, lane, eps, mean, rstd);
    if (lane == 0) stats[item] = make_float2(mean, rstd);
}

// One warp writes the merged-operand rows of up to two items (dst0 / dst1, C bf16 each)
// from the patch rows src0 / src1 of bf16 features x (-1: a pad position, zeros; a null
// dst: no item): LayerNorm'd when has_ln, else copied. Both rows are loaded into registers
// before either is computed, so two rows' loads are in flight per warp. The arithmetic is
// the LayerNorm kernels' (same operations in the same order), so the values match theirs
// bit for bit. For C <= 32 * FUSED_VEC * 8 channels.
constexpr int FUSED_VEC = 5;
__device__ __forceinline__ void ln_rows_bf16_x2(const __nv_bfloat16* __restrict__ x, int64_t src0, int64_t src1,
                                                int C, int lane, const float* __restrict__ gamma,
                                                const float* __restrict__ beta, float eps, int has_ln,
                                                uint4* __restrict__ dst0, uint4* __restrict__ dst1) {
    const int nvec = C / 8;
    uint4 u[2][FUSED_VEC];
    const int64_t src[2] = {src0, src1};
    uint4* dst[2] = {dst0, dst1};
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < FUSED_VEC; ++i) {
            const int v = lane + 32 * i;
            u[t][i] = (dst[t] != nullptr && src[t] >= 0 && v < nvec)
                          ? __ldg(reinterpret_cast<const uint4*>(x + src[t] * C) + v)
                          : make_uint4(0, 0, 0, 0);
        }
    const float inv_c = 1.0f / static_cast<float>(C);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        if (dst[t] == nullptr) continue;                        // warp-uniform
        if (src[t] < 0 || !has_ln) {                            // pad: zeros; no LayerNorm: the bf16 row
#pragma unroll
            for (int i = 0; i < FUSED_VEC; ++i)
                if (lane + 32 * i < nvec) dst[t][lane + 32 * i] = u[t][i];
            continue;
        }
        uint64_t q[FUSED_VEC][4];
#pragma unroll
        for (int i = 0; i < FUSED_VEC; ++i) {
            const uint32_t w[4] = {u[t][i].x, u[t][i].y, u[t][i].z, u[t][i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) q[i][e] = f2_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
        }
        uint64_t acc = 0;
#pragma unroll
        for (int i = 0; i < FUSED_VEC; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc = f2_add(acc, q[i][e]);
        const float mean = ln_warp_total(acc) * inv_c;
        const uint64_t nm = f2_splat(-mean);
        acc = 0;
#pragma unroll
        for (int i = 0; i < FUSED_VEC; ++i) {
            if (lane + 32 * i < nvec) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    q[i][e] = f2_add(q[i][e], nm);
                    acc = f2_fma(q[i][e], q[i][e], acc);
                }
            }
        }
        const float rstd = rsqrtf(ln_warp_total(acc) * inv_c + eps);
        const uint64_t r2 = f2_splat(rstd);
#pragma unroll
        for (int i = 0; i < FUSED_VEC; ++i) {
            const int v = lane + 32 * i;
            if (v >= nvec) continue;
            const float4* g4 = reinterpret_cast<const float4*>(gamma) + 2 * v;
            const float4* b4 = reinterpret_cast<const float4*>(beta) + 2 * v;
            dst[t][v] = ln_out_pairs(q[i], r2, __ldg(g4), __ldg(g4 + 1), __ldg(b4), __ldg(b4 + 1));
        }
    }
}

// Pipelined form for C <= 256 * kVec. Items are dealt to warps with a stride of the
// grid's warp count; each warp keeps up to `stages` of its next patch rows in flight in
// a shared-memory ring of its own, fetched by 1D bulk copies that complete on one
// mbarrier per slot, so a grid of resident blocks keeps the memory system busy while
// the warps normalise. A row is read from its slot once into registers (kVec vectors of
// 4 packed pairs per lane). gamma / beta are staged once per block in shared memory as
// four arrays of float4 (channels 8v..8v+3 and 8v+4..8v+7 of each), so that a warp's
// reads of one of them are consecutive. A wait that runs out latches
// VLPROJ_ERR_TIMEOUT in *err, waits for the warp's copies still in flight (bounded by
// LNP_DRAIN_NS, not by the wait bound) and ends the warp. Shared memory: LNP_BAR_BYTES,
// then 8 C bytes of gamma / beta when has_ln, then the rings.
constexpr int LNP_WARPS = 8;
constexpr int LNP_MAX_STAGES = 16;
constexpr int LNP_BAR_BYTES = LNP_WARPS * LNP_MAX_STAGES * 8;
constexpr uint64_t LNP_DRAIN_NS = 1000000000ull;

template <bool kF32In, int kVec>
static __global__ void __launch_bounds__(LNP_WARPS * 32, kVec > 5 ? 2 : 3) vlp_ln_merge_pipe_kernel(
    const void* __restrict__ x, const ViewDesc* __restrict__ views, int n_views, int M, int k, int C,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps, int has_ln,
    __nv_bfloat16* __restrict__ A, int stages,
    uint64_t wait_ns, int* err) {
    extern __shared__ __align__(128) uint8_t lnp_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int kk = k * k;
    const int nvec = C / 8;
    const int64_t total = static_cast<int64_t>(M) * kk;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * LNP_WARPS;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * LNP_WARPS + warp;
    float4* gb = reinterpret_cast<float4*>(lnp_smem + LNP_BAR_BYTES);     // [4][nvec]
    if (has_ln) {
        for (int v = threadIdx.x; v < nvec; v += LNP_WARPS * 32) {
            const float4* g4 = reinterpret_cast<const float4*>(gamma) + 2 * v;
            const float4* b4 = reinterpret_cast<const float4*>(beta) + 2 * v;
            gb[v] = __ldg(g4);
            gb[nvec + v] = __ldg(g4 + 1);
            gb[2 * nvec + v] = __ldg(b4);
            gb[3 * nvec + v] = __ldg(b4 + 1);
        }
    }
    __syncthreads();
    if (gw >= total) return;
    const int n_items = static_cast<int>((total - gw + nwarps - 1) / nwarps);
    const uint32_t row_bytes = static_cast<uint32_t>(C) * (kF32In ? 4u : 2u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(lnp_smem) + warp * LNP_MAX_STAGES;
    uint8_t* ring = lnp_smem + LNP_BAR_BYTES + (has_ln ? 8 * C : 0) + static_cast<size_t>(warp) * stages * row_bytes;
    const uint8_t* xb = static_cast<const uint8_t*>(x);
    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    // Lane l holds the source row of the warp's item (32 b + l), -1 for a zero pad.
    int64_t batch_row = -1;
    uint32_t loaded = 0, phase = 0;     // per slot: a copy was issued / parity to wait for
    int si = 0;                         // slot of the next issue (j mod stages)
    auto issue = [&](int j) {           // warp-uniform, called for j = 0, 1, 2, ... in order
        const int s = si;
        si = si + 1 == stages ? 0 : si + 1;
        if (j >= n_items) {
            loaded &= ~(1u << s);
            return;
        }
        if ((j & 31) == 0) {
            batch_row = -1;
            if (j + lane < n_items) {
                const int64_t it = gw + static_cast<int64_t>(j + lane) * nwarps;
                const int m = static_cast<int>(it / kk);
                batch_row =
                    merge_source_row(views, n_views, m, static_cast<int>(it - static_cast<int64_t>(m) * kk), k);
            }
        }
        const int64_t r = __shfl_sync(0xffffffffu, batch_row, j & 31);
        if (r >= 0) {
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[s], row_bytes);
                bulk_load_1d(ring + static_cast<size_t>(s) * row_bytes, xb + r * row_bytes, row_bytes, &bars[s]);
            }
            loaded |= 1u << s;
        } else {
            loaded &= ~(1u << s);
        }
    };
    for (int j = 0; j < stages; ++j) issue(j);

    const uint64_t zero2 = 0;
    const float inv_c = 1.0f / static_cast<float>(C);
    const int64_t dst_step = nwarps * C / 8;            // uint4 between a warp's items
    uint4* dst = reinterpret_cast<uint4*>(A + gw * C);
    for (int j = 0, s = 0; j < n_items; ++j, s = s + 1 == stages ? 0 : s + 1, dst += dst_step) {
        if (!((loaded >> s) & 1u)) {            // neighbour outside the grid: zeros
            issue(j + stages);
            for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
            continue;
        }
        if (!mbar_wait_limit(&bars[s], (phase >> s) & 1u, wait_ns)) {
            if (lane == 0) atomicCAS(err, 0, -5);
            // drain: no copy may still be landing in the ring when the warp ends, so these
            // waits have their own, longer bound (copies of a few KB land in microseconds)
            for (int t = 0; t < stages; ++t)
                if ((loaded >> t) & 1u) mbar_wait_limit(&bars[t], (phase >> t) & 1u, LNP_DRAIN_NS);
            return;
        }
        phase ^= 1u << s;
        const uint8_t* st = ring + static_cast<size_t>(s) * row_bytes;
        uint64_t q[kVec][4];
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            if (lane + 32 * i < nvec) {
                ln_smem_pairs<kF32In>(st, lane + 32 * i, q[i]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) q[i][e] = zero2;
            }
        }
        // the slot's bytes are in registers: order those reads before the next copy into it
        fence_proxy_async_smem();
        __syncwarp();
        issue(j + stages);

        float rstd = 1.f;
        if (has_ln) {
            uint64_t acc = 0;
#pragma unroll
            for (int i = 0; i < kVec; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc = f2_add(acc, q[i][e]);
            const float mean = ln_warp_total(acc) * inv_c;
            const uint64_t nm = f2_splat(-mean);
            acc = 0;
#pragma unroll
            for (int i = 0; i < kVec; ++i) {
                if (lane + 32 * i < nvec) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        q[i][e] = f2_add(q[i][e], nm);          // keep d = x - mean
                        acc = f2_fma(q[i][e], q[i][e], acc);
                    }
                }
            }
            rstd = rsqrtf(ln_warp_total(acc) * inv_c + eps);
        }
        const uint64_t r2 = f2_splat(rstd);
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const int v = lane + 32 * i;
            if (v >= nvec) continue;
            dst[v] = has_ln ? ln_out_pairs(q[i], r2, gb[v], gb[nvec + v], gb[2 * nvec + v], gb[3 * nvec + v])
                            : ln_convert_pairs(q[i]);
        }
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
