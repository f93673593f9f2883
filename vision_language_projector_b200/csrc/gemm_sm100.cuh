// Projector GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
//
//   GEMM1 (A from the patch features, EPI_GELU):
//       H[m, n]  = bf16( GELU( sum_q A[m, q] W1p[n, q] + b1[n] ) )
//       A is never materialised: row m of A is the k x k neighbourhood of merged
//       token m. The space-to-depth is a k x k convolution of stride k, so the A
//       tile is fetched with TMA im2col loads straight from the channel-last
//       features: for K-block (dy, dx, c0) one load walks the tile's tokens (base
//       positions (k*j, k*i) of each view, wrapping rows and views) and copies
//       channels c0..c0+63 of patch (k*i + dy, k*j + dx); patches past the grid
//       (the high-end pad) read as zero. When k divides the grid and w' divides
//       128, the same gather is one 5D tiled box (A_BOX5): the features seen as
//       (c, dx, j, dy, merged row) with strides (1, C, kC, wC, kwC) and box
//       (64, 1, w', 1, 128/w') hold a 128-token tile in token order. A_CPASYNC is
//       the gather done with 16-byte cp.async copies (zero-filled pad).
//   GEMM2 (A_TILE, EPI_SCATTER):
//       out[dest[m], n] = bf16( sum_q H[m, q] W2[n, q] + b2[n] )
//       the epilogue writes each row straight into its placeholder row.
//   Backward epilogues (A_TILE, no scatter):
//       EPI_BWD_H   P = acc + b1: G = bf16(GELU'(P)) and H = bf16(GELU(P)), row-major
//       EPI_DGELU   dP = bf16(acc * G), row-major
//   The weight gradients (K = tokens) read dY, H, dP and A row-major as MN-major operands.
//   bf16 outputs with plain rows (GEMM1's H, the backward's G, H, dP) leave the epilogue
//   as 32 x 32 blocks through shared memory and TMA tile stores.
//       EPI_F32     acc as fp32, row-major (weight and input gradients)
//       EPI_BF16    acc as bf16 through TMA stores (the LayerNorm backward's dA)
//       EPI_FOLD_F32  acc as fp32, folded back onto the patches: column p*C + c of
//                   merged token m goes to channel c of the patch at position p of its
//                   k x k neighbourhood (gmeta), so dA never goes to memory
//
// One persistent CTA (or CTA pair) per SM (pair of SMs) walks output tiles in banded
// order (see tile_coords: the CTAs running together share A tiles and an L2-sized band
// of B), statically or from a device counter (TileSeq). Roles, by warp:
//   warp 0      TMA producer (B; A in the TMA modes)
//   warp 1      TMEM allocator and the single MMA-issuing thread
//   warps 2-3   A gather producers in A_CPASYNC mode (64 threads)
//   warps 4-7   epilogue: TMEM -> registers -> bias (+GELU) -> bf16 -> global
//   warps 8-11  thread-gather / fused-producer modes, or the second epilogue group of
//               256 x 512 tiles
// Shared memory holds a STAGES-deep ring of (A, B) K-blocks of 64 bf16 (128 B
// rows, 128-byte swizzle); TMEM holds two accumulators so the epilogue of one tile
// overlaps the MMAs of the next (one, over all 512 columns, for 256 x 512 tiles).
//
// Every wait is bounded (GemmParams::wait_ns). When one runs out, the kernel
// latches VLPROJ_ERR_TIMEOUT, every role unwinds, outstanding copies and MMAs
// are drained under a separate 1 s bound, TMEM is freed, and the kernel returns.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "gelu_poly.cuh"
#include "kernels_aux.cuh"
#include "ptx.cuh"

namespace vlp {

constexpr int BM = 128;
constexpr int BK = 64;                  // 64 bf16 = one 128-byte swizzle row
constexpr int GEMM_THREADS = 256;
constexpr int GATHER_THREADS = 64;
constexpr int GEMM_THREADS_TG = 384;    // thread-gather modes: warps 8-11 fetch (and normalise) A
constexpr int TG_THREADS = 128;
constexpr int EPI_GELU = 0;
constexpr int EPI_SCATTER = 1;
constexpr int EPI_BWD_H = 2;
constexpr int EPI_DGELU = 3;
constexpr int EPI_F32 = 4;
constexpr int EPI_FOLD_F32 = 5;
constexpr int EPI_BF16 = 6;
constexpr int A_TILE = 0;               // dense row-major A, tiled TMA
constexpr int A_IM2COL = 1;             // merge-gather by TMA im2col
constexpr int A_CPASYNC = 2;            // merge-gather by cp.async
constexpr int A_BOX5 = 3;               // merge-gather by one 5D tiled TMA box (regular grids)
constexpr int A_TGATHER = 4;            // merge-gather by 128 threads' cp.async, CTA pairs allowed
constexpr int A_TGATHER_LN = 5;         // ... then the pre-merge LayerNorm applied in shared memory
constexpr int A_FUSED = 6;              // A produced inside the kernel (merge + LayerNorm / convert) by
                                        // four producer warps per CTA, read back by TMA tiles
constexpr uint64_t DRAIN_NS = 1000000000ull;
// Naps between the tests of a wait (ns): the epilogue waits a whole tile for its
// accumulator, the gather warps about one stage for a free slot or landed copies.
constexpr uint32_t EPI_NAP_NS = 256;
constexpr uint32_t GATHER_NAP_NS = 64;
constexpr int ERR_TIMEOUT = -5;

// Shared-memory plan. kCtas = 2 runs one 256-row tile on a CTA pair: each CTA holds
// its 128 rows of A and half of the BN rows of B per stage, so a stage is 32 KB and
// six stages fit.
// Epilogues that send bf16 tiles out by TMA store stage them here, per epilogue warp in
// 32 x 32 bf16 blocks: GELU two (two chunks in flight), DGELU one (a chunk of dP), BWD_H
// two (a chunk of G and of H). SCATTER stages 32 rows x 64 columns (the two blocks side
// by side) so that its stores write whole row segments.
constexpr int EPI_BLOCK_BYTES = 32 * 32 * 2;
__host__ __device__ constexpr int epi_blocks(int epi) {
    return epi == EPI_DGELU ? 1 : (epi == EPI_GELU || epi == EPI_BWD_H || epi == EPI_BF16 || epi == EPI_SCATTER) ? 2 : 0;
}
__host__ __device__ constexpr int epi_stage_bytes(int epi) { return 4 * epi_blocks(epi) * EPI_BLOCK_BYTES; }

// Slots of the ring that hands tile indices from the TMA producer to the other roles
// (dynamic tile order).
constexpr int SCHED_SLOTS = 8;

// kAuxBytes: bytes per stage beside the operands (the LayerNorm statistics of the stage's
// 128 rows in A_TGATHER_LN), kept after the ring; such layouts size the ring from the whole
// 227 KB a CTA may use.
template <int BN, int kCtas = 1, int kEpiBytes = 0, int kAuxBytes = 0>
struct GemmLayout {
    static constexpr int B_ROWS = BN / kCtas;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = B_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int RING_BUDGET = kAuxBytes ? 232448 - 1024 - 1024 - kEpiBytes : 196608;
    static constexpr int STAGES_FIT = RING_BUDGET / (STAGE_BYTES + kAuxBytes);
    static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
    static constexpr int AUX_OFFSET = STAGES * STAGE_BYTES;
    static constexpr int AUX_BYTES_PER = kAuxBytes;
    static constexpr int EPI_OFFSET = AUX_OFFSET + STAGES * kAuxBytes;
    static constexpr int BAR_OFFSET = EPI_OFFSET + kEpiBytes;
    // full_tma[S], full_gather[S], empty[S], full_local[S], tmem_full[2], tmem_empty[2], drain,
    // sched_full[SCHED_SLOTS], sched_empty[SCHED_SLOTS]
    static constexpr int NUM_BARS = 4 * STAGES + 5 + 2 * SCHED_SLOTS;
    static constexpr int MISC_OFFSET = BAR_OFFSET + NUM_BARS * 8;
    static constexpr int RING_OFFSET = MISC_OFFSET + 16;          // tile indices of the dynamic order
    static constexpr int BYTES = RING_OFFSET + 4 * SCHED_SLOTS;
    static constexpr int SMEM_ALLOC = BYTES + 1024;      // room to align the base to 1024 B
    static_assert(SMEM_ALLOC <= 232448, "a CTA may use at most 227 KB of shared memory");
    static_assert(STAGES >= 2, "at least two stages in the ring");
    // two accumulators (one tile's epilogue overlaps the next tile's MMAs), or one for
    // 256 x 512 tiles, whose accumulator spans all 512 TMEM columns
    static constexpr int NUM_ACC = 2 * BN <= 512 ? 2 : 1;
    static constexpr uint32_t TMEM_COLS = NUM_ACC * BN;
};

// Statistics bytes per stage in A_TGATHER_LN: (mean, rstd) of each of the 128 rows.
__host__ __device__ constexpr int a_aux_bytes(int amode) { return amode == A_TGATHER_LN ? BM * 8 : 0; }
__host__ __device__ constexpr bool a_thread_gather(int amode) { return amode == A_TGATHER || amode == A_TGATHER_LN; }
// Epilogue warp groups: 256 x 512 tiles drain their one accumulator with two groups of
// four warps (columns 0-255 and 256-511), since no other tile's MMAs hide that drain.
__host__ __device__ constexpr int epi_groups(int bn) { return bn == 512 ? 2 : 1; }
__host__ __device__ constexpr int gemm_threads(int amode, int bn = 256) {
    return (a_thread_gather(amode) || amode == A_FUSED || epi_groups(bn) == 2) ? GEMM_THREADS_TG : GEMM_THREADS;
}
constexpr int FUSED_BLOCK = 256;        // A_FUSED readiness granularity: rows per block (one pair tile)

struct GemmParams {
    int M;                          // rows (merged tokens, each view's run padded in im2col varlen mode)
    int N;                          // output columns
    int K;                          // reduction length, multiple of BK
    const float* bias;              // [N] fp32
    int C;                          // channels per patch; C % BK == 0
    int k;                          // merge factor
    // A_IM2COL
    const CUtensorMap* gmaps;       // per-view im2col maps in global memory, or null (one map: tmA)
    int n_gmaps;
    const int4* chunks;             // per chunk of `chunk` rows: {map, w0, h0, n0} of its first token
    int chunk;                      // rows per im2col load: 128 (one map) or 32 (per-view maps)
    // A_BOX5: features seen as (c, dx, j, dy, merged row) with box (64, 1, w', 1, 128 / w')
    int box_rows;                   // merged rows per 128-row tile (128 / w')
    // A_CPASYNC, A_TGATHER, A_TGATHER_LN
    const __nv_bfloat16* gsrc;      // bf16 patch features [P][C]
    const int2* gmeta;              // per row: {top-left patch index, (w << 16) | valid mask}
    // A_TGATHER_LN: (mean, rstd) of the patch at tap p of row m at ln_stats[p * stats_ld + m],
    // (0, 0) for a pad position or a row past M; gamma / beta [C] fp32
    const float2* ln_stats;
    int64_t stats_ld;               // a multiple of 256 rows
    const float* ln_gamma;
    const float* ln_beta;
    // A_FUSED: the producer warps write A[m][p*C + c] (bf16, row stride K) for every merged
    // token m < M and tap p: the patch at tap p of token m (found in the view table),
    // LayerNorm'd when has_ln, rounded to bf16, or zeros in the high-end pad. Items are
    // taken in (256-row block, tap, row) order from *work; ready[b * k*k + p] counts the
    // finished items of block b, tap p (256 when done, rows past M included).
    const ViewDesc* views;
    int n_views;
    const void* feat;               // features, bf16 or fp32 (feat_f32)
    int feat_f32;
    int has_ln;
    float ln_eps;
    __nv_bfloat16* a_out;
    unsigned long long* work;       // zero at launch
    uint32_t* ready;                // zero at launch, m_blocks * k*k counters
    int m_blocks;
    // output
    __nv_bfloat16* out;             // GEMM1: H; GEMM2: embeddings [out_rows][N]
    const int32_t* rowdest;         // destination row of each m (-1 = no write), or null = row m
    int64_t out_rows;               // rows of `out` (bounds guard)
    const int* fwd_status;          // nonzero = count check failed, write nothing (null = ignore)
    int tma_store;                  // EPI_GELU: rows are stored by TMA through tmC (identity rows)
    // backward epilogues (outputs through tmC, and H through tmC2 in EPI_BWD_H)
    const __nv_bfloat16* aux;       // EPI_DGELU: G = GELU'(P) [M][N] bf16
    float* outf;                    // EPI_F32: [M][N] fp32; EPI_FOLD_F32: [patches][C] fp32
    // a_mn / b_mn: the operand is MN-major, read from a row-major [K][M] (or [K][N]) matrix
    // through a 3D map (m % 64, k, m / 64) in boxes of 64 K-rows x (rows / 64) strips (the
    // weight gradients, K = tokens, read dY, H and dP where they lie); a_mn = 2: the same
    // strips by one 2D box (64 columns x 64 K-rows) each, for a matrix whose width is not a
    // multiple of 64 (columns past it read as zeros).
    int a_mn, b_mn;
    int group_n;                    // N-blocks per raster band (see tile_coords); 0 = from l2_budget
    int64_t l2_budget;              // host only: bytes of B one raster band may hold (0 = 64 MB)
    // Dynamic tile order: [0] the next tile index, [1] units that have finished taking
    // tiles; both 0 at launch, and the last unit to finish sets them back to 0. nullptr:
    // static order. Two kernels that may run at the same time never share one.
    int* tile_queue;
    int* err;                       // latched error word
    uint64_t wait_ns;               // bound on every wait
};

__device__ __forceinline__ void latch_error(int* err, int code) { atomicCAS(err, 0, code); }

// The sequence of tiles a unit (CTA or CTA pair) runs, -1 at its end.
// Static order: unit u runs tiles u, u + units, u + 2 units, ... Over hundreds of waves
// the units drift apart, and tiles that share an A block (or a B panel) no longer run
// together: each then reads the block from DRAM on its own.
// Dynamic order: the pair leader's TMA producer takes the next index from a kernel-wide
// counter as it starts a tile, so tiles start in index order whichever units run ahead.
// It publishes each index through a ring of SCHED_SLOTS in the shared memory of both CTAs
// of the pair ("slot written" barriers of each CTA); every other role reads the ring in
// the same order and frees the slot on the leader's "slot read" barrier.
struct TileSeq {
    int next, step, num;          // static order
    bool dyn;
    int* ring;                    // this CTA's ring
    uint64_t* full;               // this CTA's "slot written" barriers
    uint64_t* empty;              // "slot read" barriers (the leader's count)
    int slot;
    uint32_t ph;
};

__device__ __forceinline__ TileSeq tile_seq(int unit, int n_units, int num_tiles, bool dyn, int* ring, uint64_t* full,
                                            uint64_t* empty) {
    TileSeq q;
    q.next = unit;
    q.step = n_units;
    q.num = num_tiles;
    q.dyn = dyn;
    q.ring = ring;
    q.full = full;
    q.empty = empty;
    q.slot = 0;
    q.ph = 0;
    return q;
}

// A reader's next tile (one thread per reading warp or role). False: the wait ran out.
template <bool kPair>
__device__ __forceinline__ bool seq_take(TileSeq& q, int& tile, uint64_t lim, volatile int* abort_flag,
                                         uint32_t nap) {
    if (!q.dyn) {
        tile = q.next < q.num ? q.next : -1;
        q.next += q.step;
        return true;
    }
    if (!mbar_wait_bounded<kPair>(&q.full[q.slot], q.ph, lim, abort_flag, nap)) return false;
    tile = *reinterpret_cast<volatile int*>(q.ring + q.slot);
    if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&q.empty[q.slot]), 0));
    else mbar_arrive(&q.empty[q.slot]);
    if (++q.slot == SCHED_SLOTS) { q.slot = 0; q.ph ^= 1; }
    return true;
}

// The writer's next tile (the leader's TMA producer): take it from the counter and
// publish it to both CTAs' rings.
template <bool kPair>
__device__ __forceinline__ bool seq_publish(TileSeq& q, int* counter, int& tile, uint64_t lim,
                                            volatile int* abort_flag) {
    if (!q.dyn) {
        tile = q.next < q.num ? q.next : -1;
        q.next += q.step;
        return true;
    }
    if (!mbar_wait_bounded<kPair>(&q.empty[q.slot], q.ph ^ 1, lim, abort_flag)) return false;
    int t = atomicAdd(counter, 1);
    if (t >= q.num) t = -1;
    *reinterpret_cast<volatile int*>(q.ring + q.slot) = t;
    if constexpr (kPair) {
        st_shared_cluster_u32(mapa_shared(smem_u32(q.ring + q.slot), 1), static_cast<uint32_t>(t));
        mbar_arrive_cluster(mapa_shared(smem_u32(&q.full[q.slot]), 1));
    }
    mbar_arrive(&q.full[q.slot]);
    if (++q.slot == SCHED_SLOTS) { q.slot = 0; q.ph ^= 1; }
    tile = t;
    return true;
}

// The writer is done taking tiles (normally or not): the last unit to get here sets the
// queue back to 0 for the next kernel that uses it.
__device__ __forceinline__ void seq_finish(int* queue, int n_units) {
    __threadfence();
    if (atomicAdd(queue + 1, 1) == n_units - 1) {
        __threadfence();
        atomicExch(queue, 0);
        atomicExch(queue + 1, 0);
    }
}

// Tile order: bands of `group_n` N-blocks; inside a band the M-block advances slowest
// and the band's N-blocks fastest, so the CTAs running together share both their A
// tiles and a band of B that fits in L2 (group_n = n_tiles gives plain N-fastest order).
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int group_n, int& m_blk,
                                            int& n_blk) {
    const int band_tiles = m_tiles * group_n;
    const int band = tile / band_tiles;
    const int r = tile - band * band_tiles;
    const int n0 = band * group_n;
    const int width = min(group_n, n_tiles - n0);
    m_blk = r / width;
    n_blk = n0 + (r - m_blk * width);
}

// GELU (erf form: 0.5 x (1 + erf(x / sqrt 2))) and its derivative (Phi(x) + x phi(x))
// of two values at a time, from the FMA-only polynomials of gelu_poly.cuh with packed
// fp32 arithmetic (float32 error below 2.5e-7 and 3.5e-7). About 13 instructions per
// value: an epilogue on erff / expf takes so many issue slots from the TMA-producer and
// MMA warps sharing its schedulers that GEMM1 measured 87.5 % tensor-pipe active,
// against 94.8 % with these.
__device__ __forceinline__ void gelu2(float& x0, float& x1) {
    const uint64_t e = erf_poly2(x0 * 0.70710678118654752f, x1 * 0.70710678118654752f);
    const uint64_t hx = f2_mul(f2_pack(x0, x1), f2_splat(0.5f));
    f2_unpack(f2_fma(hx, e, hx), x0, x1);
}

__device__ __forceinline__ void gelu_grad2(float p0, float p1, float& g0, float& g1) {
    const uint64_t d = dgelu_odd_poly2(p0 * 0.70710678118654752f, p1 * 0.70710678118654752f);
    f2_unpack(f2_fma(d, f2_splat(1.0f), f2_splat(0.5f)), g0, g1);
}

// The 32 bias values of a chunk, the same for every lane: eight broadcast 16-byte loads
// (bias is 16-byte aligned and n0 a multiple of 32) instead of one load and 32 shuffles.
__device__ __forceinline__ void load_bias32(const float* bias, int n0, float (&b)[32]) {
    const float4* b4 = reinterpret_cast<const float4*>(bias + n0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 t = __ldg(b4 + q);
        b[4 * q] = t.x;
        b[4 * q + 1] = t.y;
        b[4 * q + 2] = t.z;
        b[4 * q + 3] = t.w;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Row-major 32 x 32 bf16 block in shared memory: the lane's row, 16 packed words.
__device__ __forceinline__ void write_row_block(const uint32_t (&packed)[16], uint8_t* block, int lane) {
    uint4* r4 = reinterpret_cast<uint4*>(block + lane * 64);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        r4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
}

template <int BN, int kAMode, int kEpi, int kCtas>
__global__ void __launch_bounds__(gemm_threads(kAMode, BN), 1)
    vlp_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                    const GemmParams p) {
    using L = GemmLayout<BN, kCtas, epi_stage_bytes(kEpi) * epi_groups(BN), a_aux_bytes(kAMode)>;
    constexpr int kEpiGroups = epi_groups(BN);
    constexpr int S = L::STAGES;
    constexpr bool kPair = kCtas == 2;
    constexpr bool kGatherThreads = kAMode == A_CPASYNC;
    constexpr bool kTG = a_thread_gather(kAMode);          // warps 8-11 fetch A by cp.async
    constexpr bool kLN = kAMode == A_TGATHER_LN;           // ... and normalise it in place
    constexpr bool kFused = kAMode == A_FUSED;             // warps 8-11 produce A, TMA tiles read it
    static_assert(!(kPair && kGatherThreads), "the 64-thread cp.async gather runs on single CTAs");
    static_assert(!kPair || BN == 256 || BN == 512, "CTA pairs run 256 x 256 or 256 x 512 tiles");
    static_assert(kPair || BN <= 256, "single CTAs run 128 x 128 or 128 x 256 tiles");
    // 256 x 512 tiles (GEMM1 fed by TMA im2col): two N = 256 MMAs per K step share the A
    // stage, so each im2col load feeds twice the FLOPs; each CTA stages 2 x 128 B rows
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFFSET);
    uint64_t* full_tma = bars;
    uint64_t* full_gat = bars + S;
    uint64_t* empty = bars + 2 * S;
    uint64_t* full_loc = bars + 3 * S;
    uint64_t* tmem_full = bars + 4 * S;
    uint64_t* tmem_empty = bars + 4 * S + 2;
    uint64_t* drain = bars + 4 * S + 4;
    uint64_t* sched_full = bars + 4 * S + 5;
    uint64_t* sched_empty = sched_full + SCHED_SLOTS;
    int* ring = reinterpret_cast<int*>(smem + L::RING_OFFSET);
    // readers of each ring slot: the second CTA's TMA producer, the MMA issuer, the relay
    // threads, the cp.async gather warps, the thread-gather warps, the epilogue warps
    constexpr uint32_t sched_readers = (kPair ? 1 : 0) + 1 + ((kTG && !kLN) ? kCtas : 0) + (kGatherThreads ? 2 : 0) +
                                       (kTG ? 4 * kCtas : 0) + 4 * kEpiGroups * kCtas;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFFSET);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFFSET + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = kPair ? cluster_ctarank() : 0;      // 0 = pair leader
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        // "A ready" arrivals: the 64 gather threads (A_CPASYNC); in the thread-gather modes
        // one per gather warp of every CTA (A_TGATHER_LN) or one relay thread per CTA
        const uint32_t gat_count = kGatherThreads ? GATHER_THREADS : kLN ? 4 * kCtas : kTG ? kCtas : 1;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&full_gat[s], gat_count);
            mbar_init(&empty[s], 1);
            mbar_init(&full_loc[s], TG_THREADS);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tmem_full[a], 1);
            mbar_init(&tmem_empty[a], 4 * kEpiGroups * kCtas);  // every epilogue warp of the pair
        }
        mbar_init(drain, 1);
        for (int j = 0; j < SCHED_SLOTS; ++j) {
            mbar_init(&sched_full[j], 1);
            mbar_init(&sched_empty[j], sched_readers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmB);
        if (kAMode == A_TILE || kFused || kAMode == A_BOX5 || (kAMode == A_IM2COL && p.gmaps == nullptr))
            tma_prefetch_desc(&tmA);
        if (kAMode == A_IM2COL && p.gmaps != nullptr)
            for (int i = 0; i < p.n_gmaps; ++i) tensormap_acquire(p.gmaps + i);
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, L::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (kPair) cluster_sync();        // barriers of both CTAs initialised before any remote use
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int rows_per_tile = BM * kCtas;
    const int m_tiles = (p.M + rows_per_tile - 1) / rows_per_tile;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int group_n = (p.group_n > 0 && p.group_n < n_tiles) ? p.group_n : n_tiles;
    const int kblocks = p.K / BK;
    const int cblocks = p.C / BK;
    const uint64_t lim = p.wait_ns;
    const int unit = blockIdx.x / kCtas;                      // CTA (or CTA pair) index
    const int n_units = gridDim.x / kCtas;
    const bool dyn = p.tile_queue != nullptr;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (each CTA loads its own halves)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            const int nch = (kAMode == A_IM2COL) ? BM / p.chunk : 0;
            const uint32_t expect = (kAMode == A_CPASYNC || kTG ? 0 : L::A_BYTES * kCtas) + L::B_BYTES * kCtas;
            TileSeq seq = tile_seq(unit, n_units, num_tiles, dyn, ring, sched_full, sched_empty);
            while (ok) {
                int tile;
                const bool got = leader ? seq_publish<kPair>(seq, p.tile_queue, tile, lim, abort_flag)
                                        : seq_take<kPair>(seq, tile, lim, abort_flag, 0);
                if (!got) { ok = false; break; }
                if (tile < 0) break;
                int m_blk, n_blk;
                tile_coords(tile, m_tiles, n_tiles, group_n, m_blk, n_blk);
                const int a_row_tile = m_blk * kCtas + static_cast<int>(rank);   // this CTA's 128-row slice
                int4 ch[4] = {};
                if (kAMode == A_IM2COL)
                    for (int q = 0; q < nch; ++q) ch[q] = __ldg(&p.chunks[a_row_tile * nch + q]);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1, lim, abort_flag)) { ok = false; break; }
                    if constexpr (kFused) {
                        // the first K-block of a tap: wait until the producer warps (of every
                        // CTA) have written this block's rows at that tap
                        if (kb % cblocks == 0) {
                            const int blk = (m_blk * kCtas * BM) / FUSED_BLOCK;
                            const uint32_t* flag = p.ready + blk * p.k * p.k + kb / cblocks;
                            bool got = ld_acquire_gpu(flag) >= static_cast<uint32_t>(FUSED_BLOCK);
                            if (!got) {
                                const uint64_t t0 = globaltimer_ns();
                                while (!(got = ld_acquire_gpu(flag) >= static_cast<uint32_t>(FUSED_BLOCK))) {
                                    if (*abort_flag || globaltimer_ns() - t0 > lim) break;
                                    __nanosleep(200);
                                }
                            }
                            if (!got) { ok = false; break; }
                            fence_proxy_async_global();
                        }
                    }
                    uint8_t* sa = smem + stage * L::STAGE_BYTES;
                    uint8_t* sb = sa + L::A_BYTES;
                    const int b_row = n_blk * BN + static_cast<int>(rank) * L::B_ROWS;
                    if constexpr (kPair) {
                        const uint32_t bar = mapa_shared(smem_u32(&full_tma[stage]), 0);
                        if (leader) mbar_arrive_expect_tx(&full_tma[stage], expect);
                        if (kAMode == A_TILE || kFused) {
                            if (p.a_mn == 2) {
                                for (int q = 0; q < BM / 64; ++q)
                                    tma_load_2d_pair(sa + q * 8192, &tmA, bar, (a_row_tile * (BM / 64) + q) * 64, kb * BK);
                            } else if (p.a_mn) {
                                tma_load_3d_pair(sa, &tmA, bar, 0, kb * BK, a_row_tile * (BM / 64));
                            } else {
                                tma_load_2d_pair(sa, &tmA, bar, kb * BK, a_row_tile * BM);
                            }
                        } else if (kAMode == A_BOX5) {
                            const int pos = kb / cblocks;
                            const int c0 = (kb - pos * cblocks) * BK;
                            const int dy = pos / p.k, dx = pos - dy * p.k;
                            tma_load_5d_pair(sa, &tmA, bar, c0, dx, 0, dy, a_row_tile * p.box_rows);
                        } else if (kAMode == A_IM2COL) {
                            const int pos = kb / cblocks;
                            const int c0 = (kb - pos * cblocks) * BK;
                            const int dy = pos / p.k, dx = pos - dy * p.k;
                            for (int q = 0; q < nch; ++q) {
                                const CUtensorMap* mp = p.gmaps ? p.gmaps + ch[q].x : &tmA;
                                tma_load_im2col_4d_pair(sa + q * p.chunk * 128, mp, bar, c0, ch[q].y, ch[q].z,
                                                        ch[q].w, static_cast<uint16_t>(dx), static_cast<uint16_t>(dy));
                            }
                        }
                        if constexpr (BN == 512) {
                            // this CTA's 128 rows of each 256-column half of the tile
                            tma_load_2d_pair(sb, &tmB, bar, kb * BK, n_blk * BN + static_cast<int>(rank) * 128);
                            tma_load_2d_pair(sb + 128 * 128, &tmB, bar, kb * BK, n_blk * BN + 256 + static_cast<int>(rank) * 128);
                        } else if (p.b_mn) {
                            tma_load_3d_pair(sb, &tmB, bar, 0, kb * BK, b_row / 64);
                        } else {
                            tma_load_2d_pair(sb, &tmB, bar, kb * BK, b_row);
                        }
                    } else {
                        mbar_arrive_expect_tx(&full_tma[stage], expect);
                        if (kAMode == A_TILE || kFused) {
                            if (p.a_mn == 2) {
                                for (int q = 0; q < BM / 64; ++q)
                                    tma_load_2d(sa + q * 8192, &tmA, &full_tma[stage], (a_row_tile * (BM / 64) + q) * 64,
                                                kb * BK);
                            } else if (p.a_mn) {
                                tma_load_3d(sa, &tmA, &full_tma[stage], 0, kb * BK, a_row_tile * (BM / 64));
                            } else {
                                tma_load_2d(sa, &tmA, &full_tma[stage], kb * BK, a_row_tile * BM);
                            }
                        } else if (kAMode == A_BOX5) {
                            const int pos = kb / cblocks;
                            const int c0 = (kb - pos * cblocks) * BK;
                            const int dy = pos / p.k, dx = pos - dy * p.k;
                            tma_load_5d(sa, &tmA, &full_tma[stage], c0, dx, 0, dy, a_row_tile * p.box_rows);
                        } else if (kAMode == A_IM2COL) {
                            const int pos = kb / cblocks;                  // (dy, dx) position index
                            const int c0 = (kb - pos * cblocks) * BK;
                            const int dy = pos / p.k, dx = pos - dy * p.k;
                            for (int q = 0; q < nch; ++q) {
                                const CUtensorMap* mp = p.gmaps ? p.gmaps + ch[q].x : &tmA;
                                tma_load_im2col_4d(sa + q * p.chunk * 128, mp, &full_tma[stage], c0, ch[q].y, ch[q].z,
                                                   ch[q].w, static_cast<uint16_t>(dx), static_cast<uint16_t>(dy));
                            }
                        }
                        if (p.b_mn) tma_load_3d(sb, &tmB, &full_tma[stage], 0, kb * BK, b_row / 64);
                        else tma_load_2d(sb, &tmB, &full_tma[stage], kb * BK, b_row);
                    }
                    ++issued;
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
            if (dyn && leader) seq_finish(p.tile_queue, n_units);
            if (!ok) {
                *abort_flag = 1;
                latch_error(p.err, ERR_TIMEOUT);
            }
            if (!kPair || leader) {
                // Drain: the (at most S) most recent loads may still be landing if the MMA
                // side stopped early; in a normal run these phases are already complete.
                int st = stage;
                uint32_t ph = phase;
                const int outstanding = issued < S ? issued : S;
                for (int i = 0; i < outstanding; ++i) {
                    if (st == 0) { st = S - 1; ph ^= 1; } else { --st; }
                    volatile int never = 0;
                    mbar_wait_bounded(&full_tma[st], ph, DRAIN_NS, &never);
                }
            } else if (!ok) {
                // The second CTA's loads complete on the leader's barriers, which it cannot
                // poll: after an early stop give any copy still landing ample time.
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 200000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (the pair leader's lane 0)
        if (lane == 0 && leader) {
            constexpr int MMA_N = BN > 256 ? 256 : BN;           // N of one MMA instruction
            const uint32_t idesc = idesc_bf16_f32(BM * kCtas, MMA_N) | (p.a_mn ? IDESC_A_MN : 0u) |
                                   (p.b_mn ? IDESC_B_MN : 0u);
            // a 16-deep K slice: 32 bytes further along a K-major row, 2 KB (two 8-row
            // atoms) further down an MN-major strip
            const uint32_t a_step = p.a_mn ? 2048u : 32u, b_step = p.b_mn ? 2048u : 32u;
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            TileSeq seq = tile_seq(unit, n_units, num_tiles, dyn, ring, sched_full, sched_empty);
            while (ok) {
                int tile;
                if (!seq_take<kPair>(seq, tile, lim, abort_flag, 0)) { ok = false; break; }
                if (tile < 0) break;
                if (!mbar_wait_bounded(&tmem_empty[acc], acc_phase ^ 1, lim, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&full_tma[stage], phase, lim, abort_flag)) { ok = false; break; }
                    if (kGatherThreads || kTG) {
                        if (!mbar_wait_bounded(&full_gat[stage], phase, lim, abort_flag)) { ok = false; break; }
                        fence_proxy_async_smem();
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
                    const uint32_t sb = sa + L::A_BYTES;
                    const uint64_t da = p.a_mn ? smem_desc_mn_sw128(sa) : smem_desc_sw128(sa);
                    const uint64_t db = p.b_mn ? smem_desc_mn_sw128(sb) : smem_desc_sw128(sb);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // the start address (16-byte units) is the descriptor's low field
                        const uint64_t dak = da + static_cast<uint64_t>((kk * a_step) >> 4);
                        const uint64_t dbk = db + static_cast<uint64_t>((kk * b_step) >> 4);
                        if constexpr (kPair) {
                            tc_mma_f16_pair(d_tmem, dak, dbk, idesc, (kb | kk) != 0);
                            if constexpr (BN == 512)          // second half: B rows 16 KB on, columns 256 on
                                tc_mma_f16_pair(d_tmem + 256, dak, dbk + ((128 * 128) >> 4), idesc, (kb | kk) != 0);
                        } else {
                            tc_mma_f16(d_tmem, dak, dbk, idesc, (kb | kk) != 0);
                        }
                    }
                    if constexpr (kPair) tc_commit_pair(&empty[stage], 0x3);
                    else tc_commit(&empty[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if constexpr (kPair) tc_commit_pair(&tmem_full[acc], 0x3);
                else tc_commit(&tmem_full[acc]);
                if (++acc == L::NUM_ACC) { acc = 0; acc_phase ^= 1; }
            }
            if (!ok) {
                *abort_flag = 1;
                latch_error(p.err, ERR_TIMEOUT);
            }
            // all MMAs issued by this thread are complete once `drain` flips
            if constexpr (kPair) tc_commit_pair(drain, 0x1);
            else tc_commit(drain);
            volatile int never = 0;
            mbar_wait_bounded(drain, 0, DRAIN_NS, &never);
        }
    } else if (warp < 4) {
        // ------------------------------------------------ relay (A_TGATHER): once a stage's
        // cp.async copies of this CTA have landed, make them visible to the tensor cores'
        // proxy and tell the pair leader's MMA thread
        if (kTG && !kLN && warp == 2 && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint32_t gat_leader = kPair ? mapa_shared(smem_u32(&full_gat[0]), 0) : 0u;
            TileSeq seq = tile_seq(unit, n_units, num_tiles, dyn, ring, sched_full, sched_empty);
            while (ok) {
                int tile;
                if (!seq_take<kPair>(seq, tile, lim, abort_flag, GATHER_NAP_NS)) { ok = false; break; }
                if (tile < 0) break;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait_bounded(&full_loc[stage], phase, lim, abort_flag, GATHER_NAP_NS)) { ok = false; break; }
                    fence_proxy_async_smem();
                    if constexpr (kPair) mbar_arrive_cluster(gat_leader + 8u * static_cast<uint32_t>(stage));
                    else mbar_arrive(&full_gat[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                latch_error(p.err, ERR_TIMEOUT);
            }
        }
        // ------------------------------------------------ A gather producers (A_CPASYNC)
        if (kGatherThreads) {
            const int gt = threadIdx.x - 64;          // 0..63
            const int chunk = gt & 7;                 // 16-byte chunk of the 128-byte row
            const int rsub = gt >> 3;                 // rows rsub, rsub+8, ..., rsub+120
            const uint32_t swz = static_cast<uint32_t>((chunk ^ rsub) * 16);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            TileSeq seq = tile_seq(unit, n_units, num_tiles, dyn, ring, sched_full, sched_empty);
            while (ok) {
                // lane 0 of each of the two warps reads the ring, its warp follows
                int tile = 0, got = 1;
                if ((threadIdx.x & 31) == 0) got = seq_take<kPair>(seq, tile, lim, abort_flag, GATHER_NAP_NS) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                tile = __shfl_sync(0xffffffffu, tile, 0);
                if (!got) { ok = false; break; }
                if (tile < 0) break;
                int m_blk, n_blk;
                tile_coords(tile, m_tiles, n_tiles, group_n, m_blk, n_blk);
                int base[16];
                uint32_t wm[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int m = m_blk * BM + rsub + 8 * q;
                    if (m < p.M) {
                        const int2 g = __ldg(&p.gmeta[m]);
                        base[q] = g.x;
                        wm[q] = static_cast<uint32_t>(g.y);
                    } else {
                        base[q] = 0;
                        wm[q] = 0;
                    }
                }
                for (int kb = 0; kb < kblocks; ++kb) {
                    const int pos = kb / cblocks;
                    const int c0 = (kb - pos * cblocks) * BK + chunk * 8;
                    const int dy = pos / p.k, dx = pos - dy * p.k;
                    // one lane per warp waits, the warp follows it
                    int got = 0;
                    if ((threadIdx.x & 31) == 0)
                        got = mbar_wait_bounded(&empty[stage], phase ^ 1, lim, abort_flag, GATHER_NAP_NS) ? 1 : 0;
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) { ok = false; break; }
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int r = rsub + 8 * q;
                        const int w = static_cast<int>(wm[q] >> 16);
                        const bool valid = (wm[q] >> pos) & 1u;
                        const int64_t prow = static_cast<int64_t>(base[q]) + dy * w + dx;
                        const __nv_bfloat16* src = valid ? p.gsrc + prow * p.C + c0 : p.gsrc;
                        cp_async_16(sa + r * 128 + swz, src, valid ? 16u : 0u);
                    }
                    cp_async_arrive_noinc(&full_gat[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                latch_error(p.err, ERR_TIMEOUT);
            }
            cp_async_wait_all();
        }
    } else if (kTG && warp >= 8) {
        // ------------------------------------------------ thread gather (A_TGATHER[_LN], warps 8-11)
        // Thread t copies 16-byte chunk (t & 7) of rows (t >> 3) + 16 i, i < 8, of every A
        // stage with cp.async (a zero-filled chunk where the neighbour lies in the pad or the
        // row is past M), into the 128-byte-swizzled place the tensor cores read. In
        // A_TGATHER_LN the first 64 threads also copy the stage's (mean, rstd) pairs, and
        // the warps normalise each stage in place once it has landed, LOOK stages behind the
        // copies: y = bf16(((x - mean) * rstd) * gamma + beta) with packed fp32 arithmetic
        // (the same operations, in the same order, as the LayerNorm kernels), exactly 0 at
        // a pad position. Then every lane fences its shared-memory writes to the async
        // proxy and lane 0 of each warp arrives on the pair leader's "A ready" barrier.
        if constexpr (kTG) {
            constexpr int LOOK = S - 2 > 0 ? S - 2 : 1;
            const int gt = threadIdx.x - 256;
            const int chunk = gt & 7;
            const int rsub = gt >> 3;                                 // rows rsub + 16 i
            const uint32_t swz = static_cast<uint32_t>((chunk ^ (rsub & 7)) * 16);
            const uint32_t gat_leader = kPair ? mapa_shared(smem_u32(&full_gat[0]), 0) : 0u;
            int stage = 0, tstage = 0, tkb = 0;
            uint32_t phase = 0, tphase = 0;
            int pending = 0;
            bool ok = true;
            // normalise the oldest issued stage in place and hand it to the MMA
            auto transform_one = [&]() -> bool {
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_loc[tstage], tphase, lim, abort_flag, GATHER_NAP_NS)))
                    return false;
                uint8_t* sa = smem + tstage * L::STAGE_BYTES;
                const float2* st = reinterpret_cast<const float2*>(smem + L::AUX_OFFSET + tstage * L::AUX_BYTES_PER);
                const int c0 = (tkb - (tkb / cblocks) * cblocks) * BK + chunk * 8;
                const float4 g0 = __ldg(reinterpret_cast<const float4*>(p.ln_gamma + c0));
                const float4 g1 = __ldg(reinterpret_cast<const float4*>(p.ln_gamma + c0) + 1);
                const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.ln_beta + c0));
                const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.ln_beta + c0) + 1);
                const uint64_t gg[4] = {f2_pack(g0.x, g0.y), f2_pack(g0.z, g0.w), f2_pack(g1.x, g1.y),
                                        f2_pack(g1.z, g1.w)};
                const uint64_t bb[4] = {f2_pack(b0.x, b0.y), f2_pack(b0.z, b0.w), f2_pack(b1.x, b1.y),
                                        f2_pack(b1.z, b1.w)};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = rsub + 16 * i;
                    const float2 ms = st[r];
                    uint4* cell = reinterpret_cast<uint4*>(sa + r * 128 + swz);
                    uint4 u = *cell;
                    if (ms.y == 0.0f) {
                        u = make_uint4(0, 0, 0, 0);               // pad position: exact zero
                    } else {
                        const uint64_t nm = f2_splat(-ms.x), r2 = f2_splat(ms.y);
                        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint64_t d =
                                f2_add(f2_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)), nm);
                            float lo, hi;
                            f2_unpack(f2_fma(f2_mul(d, r2), gg[e], bb[e]), lo, hi);
                            w[e] = pack_bf16x2(lo, hi);
                        }
                        u = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    *cell = u;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (kPair) mbar_arrive_cluster(gat_leader + 8u * static_cast<uint32_t>(tstage));
                    else mbar_arrive(&full_gat[tstage]);
                }
                if (++tstage == S) { tstage = 0; tphase ^= 1; }
                if (++tkb == kblocks) tkb = 0;
                return true;
            };
            TileSeq seq = tile_seq(unit, n_units, num_tiles, dyn, ring, sched_full, sched_empty);
            while (ok) {
                int tile = 0, got = 1;
                if (lane == 0) got = seq_take<kPair>(seq, tile, lim, abort_flag, GATHER_NAP_NS) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                tile = __shfl_sync(0xffffffffu, tile, 0);
                if (!got) { ok = false; break; }
                if (tile < 0) break;
                int m_blk, n_blk;
                tile_coords(tile, m_tiles, n_tiles, group_n, m_blk, n_blk);
                const int row0 = (m_blk * kCtas + static_cast<int>(rank)) * BM;      // this CTA's 128 rows
                int base[8];
                uint32_t wm[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = row0 + rsub + 16 * i;
                    if (m < p.M) {
                        const int2 g = __ldg(&p.gmeta[m]);
                        base[i] = g.x;
                        wm[i] = static_cast<uint32_t>(g.y);
                    } else {
                        base[i] = 0;
                        wm[i] = 0;
                    }
                }
                for (int kb = 0; kb < kblocks; ++kb) {
                    const int pos = kb / cblocks;
                    const int c0 = (kb - pos * cblocks) * BK + chunk * 8;
                    const int dy = pos / p.k, dx = pos - dy * p.k;
                    int got = 0;
                    if (lane == 0)
                        got = mbar_wait_bounded(&empty[stage], phase ^ 1, lim, abort_flag, GATHER_NAP_NS) ? 1 : 0;
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) { ok = false; break; }
                    const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = rsub + 16 * i;
                        const int w = static_cast<int>(wm[i] >> 16);
                        const bool valid = (wm[i] >> pos) & 1u;
                        const int64_t prow = static_cast<int64_t>(base[i]) + dy * w + dx;
                        const __nv_bfloat16* src = valid ? p.gsrc + prow * p.C + c0 : p.gsrc;
                        cp_async_16(sa + r * 128 + swz, src, valid ? 16u : 0u);
                    }
                    if constexpr (kLN) {
                        if (gt < 64) {      // the stage's statistics, two rows per thread
                            const float2* src = p.ln_stats + static_cast<int64_t>(pos) * p.stats_ld + row0 + 2 * gt;
                            cp_async_16(smem_u32(smem + L::AUX_OFFSET + stage * L::AUX_BYTES_PER) + 16 * gt, src, 16u);
                        }
                    }
                    cp_async_arrive_noinc(&full_loc[stage]);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                    if constexpr (kLN) {
                        if (++pending > LOOK) {
                            if (!transform_one()) { ok = false; break; }
                            --pending;
                        }
                    }
                }
            }
            if constexpr (kLN) {
                while (ok && pending > 0) {
                    if (!transform_one()) { ok = false; break; }
                    --pending;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                latch_error(p.err, ERR_TIMEOUT);
            }
            cp_async_wait_all();
        }
    } else if (warp >= 8 && kEpiGroups == 1) {
        // ------------------------------------------------ A producers (A_FUSED, warps 8-11)
        // Each warp takes two items at a time from the kernel-wide counter, in (256-row
        // block, tap, row) order, so the blocks become ready in the order the tiles need
        // them, whichever CTAs are running. Item (b, p, r) is merged token m = 256 b + r
        // at tap p: its patch row, LayerNorm'd (or converted), lands at A[m][p*C ...].
        // Every lane fences its writes to the async proxy (TMA loads will read them), then
        // lane 0 adds the items to their blocks' counters with release semantics.
        if constexpr (kFused) {
            const int kk = p.k * p.k;
            const uint64_t per_block = static_cast<uint64_t>(FUSED_BLOCK) * kk;
            const uint64_t total = static_cast<uint64_t>(p.m_blocks) * per_block;
            const bool fast = !p.feat_f32 && p.C <= 32 * FUSED_VEC * 8;
            const int K = p.K;
            while (!*abort_flag) {
                unsigned long long j0 = 0;
                if (lane == 0) j0 = atomicAdd(p.work, 2ull);
                j0 = __shfl_sync(0xffffffffu, j0, 0);
                if (j0 >= total) break;
                int64_t src[2] = {-1, -1};
                uint4* dst[2] = {nullptr, nullptr};
                uint32_t* cnt[2] = {nullptr, nullptr};
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint64_t j = j0 + t;
                    if (j >= total) continue;
                    const int b = static_cast<int>(j / per_block);
                    const int rem = static_cast<int>(j - static_cast<uint64_t>(b) * per_block);
                    const int pp = rem / FUSED_BLOCK;
                    const int m = b * FUSED_BLOCK + (rem - pp * FUSED_BLOCK);
                    cnt[t] = p.ready + b * kk + pp;
                    if (m >= p.M) continue;                      // rows past M: nothing to write
                    src[t] = merge_source_row(p.views, p.n_views, m, pp, p.k);
                    dst[t] = reinterpret_cast<uint4*>(p.a_out + static_cast<int64_t>(m) * K + pp * p.C);
                }
                if (fast) {
                    ln_rows_bf16_x2(static_cast<const __nv_bfloat16*>(p.feat), src[0], src[1], p.C, lane, p.ln_gamma,
                                    p.ln_beta, p.ln_eps, p.has_ln, dst[0], dst[1]);
                } else {
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (dst[t] == nullptr) continue;
                        if (src[t] < 0) {
                            for (int v = lane; v < p.C / 8; v += 32) dst[t][v] = make_uint4(0, 0, 0, 0);
                        } else if (p.feat_f32) {
                            ln_row_write<true>(p.feat, src[t], p.C, lane, p.ln_gamma, p.ln_beta, p.ln_eps, p.has_ln,
                                               dst[t]);
                        } else {
                            ln_row_write<false>(p.feat, src[t], p.C, lane, p.ln_gamma, p.ln_beta, p.ln_eps, p.has_ln,
                                                dst[t]);
                        }
                    }
                }
                fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) {
                    if (cnt[0]) red_release_gpu_add(cnt[0], 1u);
                    if (cnt[1]) red_release_gpu_add(cnt[1], 1u);
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 4..7 of each CTA)
        const int ew = warp & 3;                      // TMEM lanes 32*ew .. 32*ew+31
        const int eg = kEpiGroups == 2 ? (warp >> 3) : 0;   // column group (warps 8-11: the second)
        uint8_t* ebuf = smem + L::EPI_OFFSET + (eg * 4 + ew) * epi_blocks(kEpi) * EPI_BLOCK_BYTES;   // this warp's blocks
        int ehalf = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        const int status_ok = p.fwd_status ? (*p.fwd_status == 0) : 1;
        TileSeq seq = tile_seq(unit, n_units, num_tiles, dyn, ring, sched_full, sched_empty);
        while (ok) {
            // one lane reads the ring and waits, the warp follows it, so tcgen05.ld below is
            // never divergent
            int tile = 0, got = 1;
            if (lane == 0) got = seq_take<kPair>(seq, tile, lim, abort_flag, EPI_NAP_NS) ? 1 : 0;
            got = __shfl_sync(0xffffffffu, got, 0);
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (!got) { ok = false; break; }
            if (tile < 0) break;
            int m_blk, n_blk;
            tile_coords(tile, m_tiles, n_tiles, group_n, m_blk, n_blk);
            if (lane == 0) got = mbar_wait_bounded(&tmem_full[acc], acc_phase, lim, abort_flag, EPI_NAP_NS) ? 1 : 0;
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!got) { ok = false; break; }
            tc_fence_after();
            const int m_row0 = (m_blk * kCtas + static_cast<int>(rank)) * BM + ew * 32;
            const int m = m_row0 + lane;
            bool row_ok = m < p.M && status_ok;
            int64_t d = m;
            if (row_ok && p.rowdest) d = __ldg(&p.rowdest[m]);
            row_ok = row_ok && d >= 0 && d < p.out_rows;
            __nv_bfloat16* dst_row = (row_ok && p.out) ? p.out + d * p.N : nullptr;
            int2 fold = make_int2(0, 0);
            if constexpr (kEpi == EPI_FOLD_F32) {
                if (row_ok) fold = __ldg(&p.gmeta[m]);
            }
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + static_cast<uint32_t>(acc * BN);
            constexpr int kChunks = BN / 32 / kEpiGroups;      // this warp's 32-column chunks
#pragma unroll 1
            for (int c = eg * kChunks; c < (eg + 1) * kChunks; ++c) {
                const int n0 = n_blk * BN + c * 32;
                if (n0 >= p.N) break;                  // uniform across the warp
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_row + c * 32, v);
                tmem_ld_wait();
                if constexpr (kEpi == EPI_F32 || kEpi == EPI_FOLD_F32) {
                    float* dst = nullptr;
                    if constexpr (kEpi == EPI_F32) {
                        if (row_ok) dst = p.outf + static_cast<int64_t>(m) * p.N + n0;
                    } else if (row_ok) {
                        // a 32-column chunk lies inside one position: C is a multiple of 64
                        const int pos = n0 / p.C, c0 = n0 - pos * p.C;
                        const uint32_t wm = static_cast<uint32_t>(fold.y);
                        if ((wm >> pos) & 1u) {
                            const int dy = pos / p.k, dx = pos - dy * p.k;
                            const int64_t prow = static_cast<int64_t>(fold.x) + dy * static_cast<int>(wm >> 16) + dx;
                            dst = p.outf + prow * p.C + c0;
                        }
                    }
                    if (dst) {
                        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            d4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    }
                } else if constexpr (kEpi == EPI_BWD_H || kEpi == EPI_DGELU) {
                    // BWD_H: G = GELU'(P) through tmC and H = GELU(P) through tmC2; DGELU: dP =
                    // (accumulator) * G through tmC. Row-major 32 x 32 blocks through shared
                    // memory and TMA stores (rows and columns past the tensors are not written).
                    uint32_t packed[16];
                    uint32_t hp[16];
                    if constexpr (kEpi == EPI_BWD_H) {
                        float bb[32];
                        load_bias32(p.bias, n0, bb);
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            float x0 = __uint_as_float(v[j]) + bb[j];
                            float x1 = __uint_as_float(v[j + 1]) + bb[j + 1];
                            float g0, g1;
                            gelu_grad2(x0, x1, g0, g1);
                            packed[j / 2] = pack_bf16x2(g0, g1);
                            gelu2(x0, x1);
                            hp[j / 2] = pack_bf16x2(x0, x1);
                        }
                    } else {
                        uint4 g4[4] = {};
                        if (row_ok) {
                            const uint4* src = reinterpret_cast<const uint4*>(p.aux + static_cast<int64_t>(m) * p.N + n0);
#pragma unroll
                            for (int j = 0; j < 4; ++j) g4[j] = __ldg(src + j);
                        }
                        const uint32_t* gw = reinterpret_cast<const uint32_t*>(g4);
#pragma unroll
                        for (int j = 0; j < 32; j += 2)
                            packed[j / 2] = pack_bf16x2(__uint_as_float(v[j]) * __uint_as_float(gw[j / 2] << 16),
                                                        __uint_as_float(v[j + 1]) * __uint_as_float(gw[j / 2] & 0xFFFF0000u));
                    }
                    if (lane == 0) bulk_wait_read<0>();      // the previous chunk's stores have read the blocks
                    __syncwarp();
                    write_row_block(packed, ebuf, lane);
                    if constexpr (kEpi == EPI_BWD_H) write_row_block(hp, ebuf + EPI_BLOCK_BYTES, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && m_row0 < p.M) {         // a block wholly past M is not stored
                        tma_store_2d(&tmC, ebuf, n0, m_row0);
                        if constexpr (kEpi == EPI_BWD_H) tma_store_2d(&tmC2, ebuf + EPI_BLOCK_BYTES, n0, m_row0);
                        bulk_commit_group();
                    }
                } else if constexpr (kEpi == EPI_SCATTER) {
                    // The warp's 32 rows x 64 columns (two chunks) are staged in shared memory,
                    // 128 bytes per row with the 16-byte chunk index XOR (row & 7), so both the
                    // row-wise writes below and the column-wise reads after them touch every
                    // bank once per 128 bytes. Then each store instruction writes 4 rows x 128
                    // contiguous bytes: lane l takes 16-byte chunk (l & 7) of row 4 i + (l >> 3),
                    // sent to that row's placeholder row (lanes share the destinations by shuffle).
                    float bb[32];
                    load_bias32(p.bias, n0, bb);
                    const int half = c & 1;
                    if (half == 0) __syncwarp();             // the previous block has been read out
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2)
                        packed[j / 2] = pack_bf16x2(__uint_as_float(v[j]) + bb[j], __uint_as_float(v[j + 1]) + bb[j + 1]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int q = half * 4 + j;
                        *reinterpret_cast<uint4*>(ebuf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                    }
                    if (half == 1 || c + 1 == (eg + 1) * kChunks || n0 + 32 >= p.N) {
                        __syncwarp();
                        const int nb = n0 - half * 32;               // first column of the block
                        const int q = lane & 7;
                        const bool col_ok = q < 4 * (half + 1);      // a lone last chunk fills q < 4
                        const int64_t my_dest = row_ok ? d : -1;
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int r = 4 * it + (lane >> 3);
                            const int64_t dr = __shfl_sync(0xffffffffu, my_dest, r);
                            if (dr >= 0 && col_ok) {
                                const uint4 val = *reinterpret_cast<const uint4*>(ebuf + r * 128 + ((q ^ (r & 7)) << 4));
                                *reinterpret_cast<uint4*>(p.out + dr * p.N + nb + q * 8) = val;
                            }
                        }
                    }
                } else {
                    float bb[32];
                    if constexpr (kEpi == EPI_BF16) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) bb[j] = 0.0f;
                    } else {
                        load_bias32(p.bias, n0, bb);
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float x0 = __uint_as_float(v[j]) + bb[j];
                        float x1 = __uint_as_float(v[j + 1]) + bb[j + 1];
                        if (kEpi == EPI_GELU) gelu2(x0, x1);
                        packed[j / 2] = pack_bf16x2(x0, x1);
                    }
                    if ((kEpi == EPI_GELU || kEpi == EPI_BF16) && p.tma_store) {
                        // rows leave through a shared-memory block and one TMA store (full
                        // lines, instead of 32 rows touched per store instruction)
                        uint8_t* blk = ebuf + ehalf * EPI_BLOCK_BYTES;
                        if (lane == 0) bulk_wait_read<1>();  // the store from this block two chunks ago is done
                        __syncwarp();
                        write_row_block(packed, blk, lane);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && m_row0 < p.M) {
                            tma_store_2d(&tmC, blk, n0, m_row0);
                            bulk_commit_group();
                        }
                        ehalf ^= 1;
                    } else if (row_ok) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst_row + n0);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&tmem_empty[acc]), 0));
                else mbar_arrive(&tmem_empty[acc]);
            }
            if (++acc == L::NUM_ACC) { acc = 0; acc_phase ^= 1; }
        }
        if (!ok) {
            *abort_flag = 1;
            latch_error(p.err, ERR_TIMEOUT);
        }
        if constexpr (epi_stage_bytes(kEpi) > 0) {
            if (lane == 0) bulk_wait_all();          // every TMA store of this warp has landed
            __syncwarp();
        }
    }

    __syncwarp();                     // lanes that skipped a role rejoin their lane 0
    tc_fence_before();
    // A pair's CTAs read each other's shared memory (MMA operands, barriers): neither
    // leaves before the other is done.
    if constexpr (kPair) cluster_sync();
    else __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        if constexpr (kPair) tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
        else tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

}  // namespace vlp
