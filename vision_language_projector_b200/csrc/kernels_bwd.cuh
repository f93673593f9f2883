// Memory-bound kernels of the projector backward (sm_100a):
//   gather-transpose   rows of a bf16 matrix, optionally picked through a row table,
//                      copied row-major and / or transposed through shared memory
//                      (dY from the output gradient, the transposed weights)
//   column sums        bias gradients: row-block partials of dY and dP, then the
//                      blocks added in order
//   dW1 reorder        dW1's columns from the kernel's K order to the caller's
//   LayerNorm backward input gradient per patch, gamma / beta partial sums per block
//                      (without a LayerNorm the dA GEMM's epilogue writes the input
//                      gradient itself)
//   column sums        gamma / beta (and newline / separator) gradients from partials
//   special-row grads  per-image newline / separator sums (2D tiling)
// Every reduction runs in a fixed order over a fixed grid, so repeated calls give the
// same bits.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels_aux.cuh"

namespace vlp {

constexpr int TR_TILE = 64;
constexpr int LNB_WARPS = 8;

// Source row m (< M) is src + sel(m) * ld_src, sel(m) = rowsel[m] when rowsel is given
// (an entry outside [0, src_rows) reads zeros) or m. When *zero_if != 0 every row
// reads zeros. Writes, for q < Q:
//   dst[m * Q + q]           row-major copy (skipped when dst is null)
//   dst_t[perm(q) * ldt + m] transposed copy (skipped when dst_t is null), where
//                            perm(q) = c*kk + p for q = p*C + c when chan_outer, else q
// Columns M .. ceil(M/8)*8 - 1 of the transposed copy are written as zeros. Grid
// (ceil(Q/64), ceil(M/64)), 256 threads. Q, ld_src and ldt are multiples of 8.
static __global__ void __launch_bounds__(256) vlp_gather_transpose_kernel(
    const __nv_bfloat16* __restrict__ src, int64_t ld_src, int64_t src_rows, const int32_t* __restrict__ rowsel,
    const int* __restrict__ zero_if, int M, int Q, __nv_bfloat16* __restrict__ dst, __nv_bfloat16* __restrict__ dst_t,
    int64_t ldt, int C, int kk, int chan_outer) {
    __shared__ __align__(16) __nv_bfloat16 tile[TR_TILE][TR_TILE + 8];
    const int q0 = blockIdx.x * TR_TILE;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * TR_TILE;
    const bool zero_all = zero_if != nullptr && *zero_if != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int idx = threadIdx.x + 256 * i;
        const int r = idx >> 3, v = idx & 7;
        const int64_t m = m0 + r;
        const int q = q0 + 8 * v;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (m < M && q < Q && !zero_all) {
            const int64_t srow = rowsel ? static_cast<int64_t>(__ldg(&rowsel[m])) : m;
            if (srow >= 0 && srow < src_rows) val = __ldg(reinterpret_cast<const uint4*>(src + srow * ld_src + q));
        }
        *reinterpret_cast<uint4*>(&tile[r][8 * v]) = val;
        if (dst != nullptr && m < M && q < Q) *reinterpret_cast<uint4*>(dst + m * Q + q) = val;
    }
    if (dst_t == nullptr) return;
    __syncthreads();
    // thread -> column qq of the tile and 16 consecutive rows: a warp reads 32 adjacent
    // columns of one tile row (no bank conflicts) and writes 32 bytes per output row
    const int qq = threadIdx.x & 63, mh = threadIdx.x >> 6;
    const int q = q0 + qq;
    if (q >= Q) return;
    int64_t orow = q;
    if (chan_outer && kk > 1) {
        const int pp = q / C, c = q - pp * C;
        orow = static_cast<int64_t>(c) * kk + pp;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r0 = 16 * mh + 8 * h;
        const int64_t m = m0 + r0;
        if (m >= M) break;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t lo = __bfloat16_as_ushort(tile[r0 + 2 * e][qq]);
            const uint32_t hi = __bfloat16_as_ushort(tile[r0 + 2 * e + 1][qq]);
            w[e] = lo | (hi << 16);
        }
        const int64_t off = orow * ldt + m;
        *reinterpret_cast<uint4*>(dst_t + off) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// dW1 from the kernel's K order back to the caller's: row n of src holds the columns
// position-outer (p * C + c), row n of dst channel-outer (c * kk + p). One block per (row,
// 64 channels): the kk runs of 64 are read coalesced, transposed in shared memory and
// written as one run of 64 kk values.
constexpr int UNPERM_MAX_KK = 9;
static __global__ void __launch_bounds__(64) vlp_unpermute_cols_kernel(const float* __restrict__ src,
                                                                       float* __restrict__ dst, int C, int kk) {
    __shared__ float tile[64 * UNPERM_MAX_KK];
    const int64_t K1 = static_cast<int64_t>(C) * kk;
    const int64_t row = static_cast<int64_t>(blockIdx.y) * K1;
    const int c0 = blockIdx.x * 64, t = threadIdx.x;
    for (int pp = 0; pp < kk; ++pp) tile[t * kk + pp] = src[row + static_cast<int64_t>(pp) * C + c0 + t];
    __syncthreads();
    float* out = dst + row + static_cast<int64_t>(c0) * kk;
    for (int i = t; i < 64 * kk; i += 64) out[i] = tile[i];
}

// Column sums of a row-major bf16 matrix [M][N] (N even), first pass: partial[b][n] is
// the sum of column n over rows [b CSR_ROWS, (b + 1) CSR_ROWS), in row order. A thread
// takes two adjacent columns (one 4-byte load per row), so a warp reads 128 contiguous
// bytes of each row; vlp_colsum_kernel then adds the row blocks in order (bias gradients:
// db2 over dY, db1 and the middle layers' db over dP).
constexpr int CSR_ROWS = 1024;
constexpr int CSR_THREADS = 128;
static __global__ void __launch_bounds__(CSR_THREADS) vlp_colsum_rows_kernel(const __nv_bfloat16* __restrict__ X,
                                                                             int64_t M, int N,
                                                                             float* __restrict__ partial) {
    const int n = 2 * (blockIdx.x * CSR_THREADS + threadIdx.x);
    if (n >= N) return;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * CSR_ROWS;
    const int64_t m1 = m0 + CSR_ROWS < M ? m0 + CSR_ROWS : M;
    const uint32_t* col = reinterpret_cast<const uint32_t*>(X + n);
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int64_t m = m0; m < m1; ++m) {
        const uint32_t w = __ldg(col + m * (N / 2));
        s0 += __uint_as_float(w << 16);
        s1 += __uint_as_float(w & 0xFFFF0000u);
    }
    float* row = partial + static_cast<int64_t>(blockIdx.y) * N;
    row[n] = s0;
    row[n + 1] = s1;
}

template <bool kF32In>
__device__ __forceinline__ void load8_feat(const void* x, int64_t row, int C, int v, float (&f)[8]) {
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
}

__device__ __forceinline__ void load8_f32(const float* p, int v, float (&f)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p) + 2 * v);
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 2 * v + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Backward of the pre-merge LayerNorm, one warp per (merged token m, position p) item as
// in the merge pass; the item's patch is row gmeta[m].x + dy * w + dx of the features,
// and items in the pad are skipped.
//   dsrc = dA[m][p*C .. p*C + C)            bf16, position-outer columns
//   xhat = (x - mean) * rstd                the forward pass's fp32 statistics
//   dx   = rstd * (g - mean(g) - xhat * mean(g * xhat)),  g = dsrc * gamma
// Each lane holds its kVec 8-channel vectors of x and dsrc in registers, so both are
// read once. dfeat [P][C] fp32 (null = not wanted) receives dx. Each warp adds
// dsrc * xhat and dsrc into its own shared-memory slice (channel 8v + e kept at
// e * C/8 + v, so the lanes of a warp hit adjacent banks), and each block writes the sum
// of its slices, in warp order, to partial[block][0 | 1][C] (null = not wanted). Items
// are dealt round-robin over a fixed grid. C <= 256 * kVec. Dynamic shared memory:
// 8 * 2 * C floats.
template <bool kF32In, int kVec>
__global__ void __launch_bounds__(256) vlp_ln_backward_kernel(const void* __restrict__ x,
                                                              const int2* __restrict__ gmeta, int M, int k, int C,
                                                              const float* __restrict__ gamma, float eps,
                                                              const __nv_bfloat16* __restrict__ dA,
                                                              float* __restrict__ dfeat,
                                                              float* __restrict__ partial) {
    extern __shared__ float lnb_acc[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int kk = k * k;
    const int nvec = C / 8;
    const float invC = 1.0f / static_cast<float>(C);
    float* my = lnb_acc + warp * 2 * C;
    for (int i = lane; i < 2 * C; i += 32) my[i] = 0.f;
    const int64_t items = static_cast<int64_t>(M) * kk;
    for (int64_t item = static_cast<int64_t>(blockIdx.x) * LNB_WARPS + warp; item < items;
         item += static_cast<int64_t>(gridDim.x) * LNB_WARPS) {
        const int m = static_cast<int>(item / kk), pp = static_cast<int>(item - static_cast<int64_t>(m) * kk);
        const int2 g = __ldg(&gmeta[m]);
        const uint32_t wm = static_cast<uint32_t>(g.y);
        if (!((wm >> pp) & 1u)) continue;
        const int dy = pp / k, dx = pp - dy * k;
        const int64_t row = static_cast<int64_t>(g.x) + dy * static_cast<int>(wm >> 16) + dx;
        const int64_t drow = static_cast<int64_t>(m) * kk + pp;     // dA row of C values
        float f[kVec][8], dd[kVec][8];
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const int v = lane + 32 * i;
            if (v < nvec) {
                load8_feat<kF32In>(x, row, C, v, f[i]);
                load8_feat<false>(dA, drow, C, v, dd[i]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) f[i][e] = dd[i][e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) s += f[i][e];
        }
        const float mean = warp_sum(s) * invC;
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            if (lane + 32 * i < nvec) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float t = f[i][e] - mean;
                    q += t * t;
                }
            }
        }
        const float rstd = rsqrtf(warp_sum(q) * invC + eps);
        float sg = 0.f, sgx = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const int v = lane + 32 * i;
            if (v >= nvec) continue;
            float gm[8];
            load8_f32(gamma, v, gm);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float xh = (f[i][e] - mean) * rstd;
                my[e * nvec + v] += dd[i][e] * xh;
                my[C + e * nvec + v] += dd[i][e];
                f[i][e] = xh;                       // x is not needed again
                dd[i][e] *= gm[e];                  // g = dsrc * gamma
                sg += dd[i][e];
                sgx += dd[i][e] * xh;
            }
        }
        if (dfeat == nullptr) continue;
        const float mg = warp_sum(sg) * invC, mgx = warp_sum(sgx) * invC;
        float* out = dfeat + row * C;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const int v = lane + 32 * i;
            if (v >= nvec) continue;
            float r[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = rstd * (dd[i][e] - mg - f[i][e] * mgx);
            reinterpret_cast<float4*>(out)[2 * v] = make_float4(r[0], r[1], r[2], r[3]);
            reinterpret_cast<float4*>(out)[2 * v + 1] = make_float4(r[4], r[5], r[6], r[7]);
        }
    }
    if (partial == nullptr) return;      // uniform over the block
    __syncthreads();
    for (int i = threadIdx.x; i < 2 * C; i += blockDim.x) {
        const int part = i >= C ? 1 : 0, c = i - part * C;
        const int slot = part * C + (c & 7) * nvec + (c >> 3);
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < LNB_WARPS; ++w) t += lnb_acc[w * 2 * C + slot];
        partial[static_cast<int64_t>(blockIdx.x) * 2 * C + i] = t;
    }
}

// out0[c] = sum over b < nb of partial[b][0][c]; out1 likewise from partial[b][1].
// A block covers 32 of the 2C sums with 8 row groups (b = g, g + 8, ...), combined in
// group order, so the result does not depend on timing.
constexpr int CS_COLS = 32;
constexpr int CS_GROUPS = 8;
static __global__ void __launch_bounds__(CS_COLS * CS_GROUPS) vlp_colsum_kernel(const float* __restrict__ partial,
                                                                               int nb, int C,
                                                                               float* __restrict__ out0,
                                                                               float* __restrict__ out1) {
    __shared__ float red[CS_GROUPS][CS_COLS];
    const int col = threadIdx.x % CS_COLS, grp = threadIdx.x / CS_COLS;
    const int c = blockIdx.x * CS_COLS + col;
    float t = 0.f;
    if (c < 2 * C)
        for (int b = grp; b < nb; b += CS_GROUPS) t += partial[static_cast<int64_t>(b) * 2 * C + c];
    red[grp][col] = t;
    __syncthreads();
    if (grp != 0 || c >= 2 * C) return;
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < CS_GROUPS; ++g) s += red[g][col];
    if (c < C) {
        if (out0) out0[c] = s;
    } else if (out1) {
        out1[c - C] = s;
    }
}

// Per image (blockIdx.y) and column n: partial[img][0][n] = sum of d_out[., n] over the
// image's newline rows, partial[img][1][n] over its separator row, rows in order (zeros
// when the count check failed). vlp_colsum_kernel then adds the images in order.
static __global__ void __launch_bounds__(256) vlp_special_grad_kernel(const ImageDesc* __restrict__ imgs,
                                                                      const int32_t* __restrict__ pos, int64_t R,
                                                                      const __nv_bfloat16* __restrict__ d_out,
                                                                      int64_t out_rows, int N,
                                                                      const int* __restrict__ fwd_status,
                                                                      float* __restrict__ partial) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float snl = 0.f, ssep = 0.f;
    if (*fwd_status == 0) {
        const ImageDesc I = imgs[blockIdx.y];
        const int n_nl = I.hp + I.th * I.hp;
        for (int s = 0; s <= n_nl; ++s) {
            const int64_t g = I.row_base + special_row(I, s);
            if (g < 0 || g >= R) continue;
            const int64_t d = pos[g];
            if (d < 0 || d >= out_rows) continue;
            const float val = __bfloat162float(d_out[d * N + n]);
            if (s < n_nl) snl += val;
            else ssep += val;
        }
    }
    float* row = partial + static_cast<int64_t>(blockIdx.y) * 2 * N;
    row[n] = snl;
    row[N + n] = ssep;
}

}  // namespace vlp
