// vlproj_backward (declared in vlproj.h): gradients of the projector for one batch.
//
// Enqueued on the caller's stream without host syncs (stage numbers as in vlproj.h):
//    6  placeholder index + geometry  placeholder positions, the count check, each merged
//                                     token's destination row and gather data
//    7  LayerNorm-merge               A [M][k*k*C] bf16, position-outer: the forward's
//                                     bf16 A operand
//    8  GEMM1 recompute               P = A W1p^T + b1 -> G = GELU'(P) and H = GELU(P),
//                                     [M][N1] bf16 each, for every hidden layer
//    9  dY gather                     dY [M][N2] from d_out's placeholder rows (zeros if
//                                     the count check failed)
//   10  dH GEMMs                      dP = (dY W2) * G -> dP [M][N1], and with depth > 2
//                                     down through the middle layers, with their weight
//                                     gradients dW_mid = dP^T H (K = M)
//   11  dW2 GEMM                      dW2 = dY^T H, K = M
//   12  dW1 GEMM                      dW1 = dP^T A, K = M, then its columns put back in
//                                     the caller's channel order
//   13  dA GEMM                       dA = dP W1p [M][k*k*C] bf16 (without a LayerNorm
//                                     folded straight onto the patches in fp32: d_features)
//   14  tails                         LayerNorm backward -> d_features and gamma / beta
//                                     partials, column sums -> dgamma, dbeta; newline /
//                                     separator gradients (db2, db1: column sums of dY and
//                                     dP, beside stages 11 and 12)
// Every contraction runs on the tcgen05 GEMM kernel with operands from tensor maps. The
// weight gradients (K = M, the tokens) read dY, H, dP and A where they lie, row-major, as
// MN-major operands; dW1's columns are then put back in the caller's order. The bias
// gradients are column sums of dY and dP over the tokens. W2^T and W1p^T are made once,
// on the first call. For batches up to about 2^28 hidden activations, stages 11-12 and
// the bias sums run on the handle's side stream, forked after stage 9 and joined before
// the call returns.
#include "host.cuh"
#include "kernels_bwd.cuh"

using namespace vlp_host;

namespace {

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Tensor maps for a B operand: box of BN rows (single CTAs) and of 128 rows (pairs).
int encode_b(CUtensorMap* full, CUtensorMap* half, const void* base, uint64_t rows, uint64_t cols, int bn,
             uint64_t ld = 0) {
    if (encode_bf16_2d(full, base, rows, cols, static_cast<uint32_t>(bn), ld)) return VLPROJ_ERR_CUDA;
    return encode_bf16_2d(half, base, rows, cols, 128, ld);
}

// A B operand read MN-major from a row-major [K][N] matrix: boxes of BN / 64 strips
// (single CTAs) and of 2 strips (each CTA of a pair holds 128 of the tile's N).
int encode_b_mn(CUtensorMap* full, CUtensorMap* half, const void* base, uint64_t rows, uint64_t cols, int bn) {
    if (encode_bf16_mn(full, base, rows, cols, static_cast<uint32_t>(bn / 64))) return VLPROJ_ERR_CUDA;
    return encode_bf16_mn(half, base, rows, cols, 2);
}

GemmParams gemm_params(const vlproj_handle* h, int64_t M, int N, int64_t K) {
    GemmParams p{};
    p.M = static_cast<int>(M);
    p.N = N;
    p.K = static_cast<int>(round_up(K, vlp::BK));
    p.C = h->cfg.C;
    p.k = h->cfg.k;
    p.out_rows = M;
    p.err = h->status;
    p.wait_ns = h->wait_ns;
    p.l2_budget = h->l2_budget;
    return p;
}

void transpose_launch(const __nv_bfloat16* src, int64_t ld_src, int64_t src_rows, const int32_t* rowsel,
                      const int* zero_if, int64_t M, int Q, __nv_bfloat16* dst, __nv_bfloat16* dst_t, int64_t ldt,
                      int C, int kk, int chan_outer, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>((Q + vlp::TR_TILE - 1) / vlp::TR_TILE),
              static_cast<unsigned>((M + vlp::TR_TILE - 1) / vlp::TR_TILE));
    vlp::vlp_gather_transpose_kernel<<<grid, 256, 0, s>>>(src, ld_src, src_rows, rowsel, zero_if,
                                                          static_cast<int>(M), Q, dst, dst_t, ldt, C, kk, chan_outer);
}

// W2^T [N1][N2], W1p^T [K1][N1] and each middle layer's W^T [N1][N1], with their tensor
// maps, made once per handle.
int ensure_transposed_weights(vlproj_handle* h, cudaStream_t s) {
    const vlproj_config& c = h->cfg;
    const size_t n1 = static_cast<size_t>(c.N1), n2 = static_cast<size_t>(c.N2), k1 = static_cast<size_t>(h->K1);
    if (!h->W2t || !h->W1pt) {
        if (!h->W2t) VLP_CUDA(cudaMalloc(&h->W2t, n1 * n2 * 2));
        if (!h->W1pt) VLP_CUDA(cudaMalloc(&h->W1pt, k1 * n1 * 2));
        h->launches += 2;
        transpose_launch(h->W2, c.N1, c.N2, nullptr, nullptr, c.N2, c.N1, nullptr, h->W2t, c.N2, c.C, 1, 0, s);
        transpose_launch(h->W1p, h->K1, c.N1, nullptr, nullptr, c.N1, h->K1, nullptr, h->W1pt, c.N1, c.C, 1, 0, s);
        VLP_CUDA(cudaGetLastError());
        if (encode_b(&h->tmW2t, &h->tmW2th, h->W2t, n1, n2, pick_bn(c.N1)) ||
            encode_b(&h->tmW1pt, &h->tmW1pth, h->W1pt, k1, n1, pick_bn(h->K1)))
            return VLPROJ_ERR_CUDA;
    }
    while (h->Wmt.size() < h->Wm.size()) {
        const size_t i = h->Wmt.size();
        __nv_bfloat16* w = nullptr;
        VLP_CUDA(cudaMalloc(&w, n1 * n1 * 2));
        h->Wmt.push_back(w);
        ++h->launches;
        transpose_launch(h->Wm[i], c.N1, c.N1, nullptr, nullptr, c.N1, c.N1, nullptr, w, c.N1, c.C, 1, 0, s);
        VLP_CUDA(cudaGetLastError());
        CUtensorMap full{}, half{};
        if (encode_b(&full, &half, w, n1, n1, pick_bn(c.N1))) return VLPROJ_ERR_CUDA;
        h->tmWmt.push_back(full);
        h->tmWmth.push_back(half);
    }
    return VLPROJ_OK;
}

int zero_outputs(const vlproj_backward_args* a, const vlproj_config& c, int K1, int64_t P, cudaStream_t s) {
    const size_t n1 = c.N1, n2 = c.N2, C = c.C;
    if (a->d_W1) VLP_CUDA(cudaMemsetAsync(a->d_W1, 0, n1 * K1 * 4, s));
    if (a->d_b1) VLP_CUDA(cudaMemsetAsync(a->d_b1, 0, n1 * 4, s));
    if (a->d_W2) VLP_CUDA(cudaMemsetAsync(a->d_W2, 0, n2 * n1 * 4, s));
    if (a->d_b2) VLP_CUDA(cudaMemsetAsync(a->d_b2, 0, n2 * 4, s));
    if (a->d_gamma) VLP_CUDA(cudaMemsetAsync(a->d_gamma, 0, C * 4, s));
    if (a->d_beta) VLP_CUDA(cudaMemsetAsync(a->d_beta, 0, C * 4, s));
    if (a->d_newline) VLP_CUDA(cudaMemsetAsync(a->d_newline, 0, n2 * 4, s));
    if (a->d_sep) VLP_CUDA(cudaMemsetAsync(a->d_sep, 0, n2 * 4, s));
    if (a->d_features && P > 0) VLP_CUDA(cudaMemsetAsync(a->d_features, 0, static_cast<size_t>(P) * C * 4, s));
    for (int i = 0; i + 2 < c.depth; ++i) {
        if (a->d_W_mid && a->d_W_mid[i]) VLP_CUDA(cudaMemsetAsync(a->d_W_mid[i], 0, n1 * n1 * 4, s));
        if (a->d_b_mid && a->d_b_mid[i]) VLP_CUDA(cudaMemsetAsync(a->d_b_mid[i], 0, n1 * 4, s));
    }
    return VLPROJ_OK;
}

bool misaligned(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 != 0; }

}  // namespace

extern "C" int vlproj_backward(vlproj_handle* h, const vlproj_backward_args* a, void* stream) {
    if (!h || !a) return VLPROJ_ERR_INVALID_ARG;
    const vlproj_config& c = h->cfg;
    if (c.has_ln && c.C > 256 * 8) return VLPROJ_ERR_UNSUPPORTED;     // LayerNorm backward keeps C in registers
    const int depth = c.depth;       // Linear layers; hidden layers 1 .. depth - 1
    const int n_mid = depth - 2;
    auto mid_w = [&](int i) -> float* { return a->d_W_mid ? a->d_W_mid[i] : nullptr; };
    auto mid_b = [&](int i) -> float* { return a->d_b_mid ? a->d_b_mid[i] : nullptr; };
    const int64_t n_ids = a->n_ids;
    if (n_ids < 0 || n_ids >= (int64_t(1) << 31)) return VLPROJ_ERR_INVALID_ARG;
    if (n_ids > 0 && (!a->input_ids || !a->d_out)) return VLPROJ_ERR_INVALID_ARG;
    if (a->n_images > 0 && !a->features) return VLPROJ_ERR_INVALID_ARG;
    for (const void* p : {a->features, a->d_out, static_cast<const void*>(a->d_W1), static_cast<const void*>(a->d_b1),
                          static_cast<const void*>(a->d_W2), static_cast<const void*>(a->d_b2),
                          static_cast<const void*>(a->d_gamma), static_cast<const void*>(a->d_beta),
                          static_cast<const void*>(a->d_newline), static_cast<const void*>(a->d_sep),
                          static_cast<const void*>(a->d_features)})
        if (misaligned(p)) return VLPROJ_ERR_INVALID_ARG;
    for (int i = 0; i < n_mid; ++i)
        if (misaligned(mid_w(i)) || misaligned(mid_b(i))) return VLPROJ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Plan pl;
    int rc = build_plan(c, a->grid_hw, a->spatial_crop, a->n_images, false, VLPROJ_GATHER_CPASYNC, &pl);
    if (rc) return rc;
    const bool tiled = c.tile_tag == VLPROJ_TILE_2D;
    const int kk = c.k * c.k;
    const int K1 = h->K1;
    const int64_t M = pl.M;          // no padding in this plan: M merged tokens
    const size_t hslab = static_cast<size_t>(M) * c.N1;
    // bias gradients: column sums over the tokens, in blocks of CSR_ROWS rows
    const int64_t nb_cs = (M + vlp::CSR_ROWS - 1) / vlp::CSR_ROWS;

    // which dP are needed: Linear l's gradients need dP_l; dP_l needs every dP above it
    const bool want_l1 = a->d_W1 || a->d_b1 || a->d_features || a->d_gamma || a->d_beta;
    const bool want_da = a->d_features || (c.has_ln && (a->d_gamma || a->d_beta));   // the dA GEMM
    int l_min = depth;               // lowest Linear whose dP is needed (dP_depth = dY)
    for (int i = n_mid - 1; i >= 0; --i)
        if (mid_w(i) || mid_b(i)) l_min = i + 2;
    if (want_l1) l_min = 1;
    const bool want_recompute = l_min < depth || a->d_W2;     // G feeds dP, H the weight gradients

    // scratch
    const int nblocks = vlp::scan_blocks(n_ids);
    if (h->counts.ensure(nblocks + 1) || h->pos.ensure(std::max<int64_t>(pl.R, 1))) return VLPROJ_ERR_CUDA;
    if (M > 0) {
        if (h->rowdest.ensure(M) || h->gmeta.ensure(M) || h->A.ensure(static_cast<size_t>(M) * K1) ||
            h->G.ensure(hslab * (depth - 1)) || h->Hr.ensure(hslab * (depth - 1)) ||
            h->dY.ensure(static_cast<size_t>(M) * c.N2) || h->dP.ensure(hslab * 2) ||
            h->part_cs.ensure(static_cast<size_t>(nb_cs) * (c.N2 + 2 * c.N1)))
            return VLPROJ_ERR_CUDA;
        if (a->d_W1 && h->dW1p.ensure(static_cast<size_t>(c.N1) * K1)) return VLPROJ_ERR_CUDA;
        if (want_da && c.has_ln && h->dA.ensure(static_cast<size_t>(M) * K1)) return VLPROJ_ERR_CUDA;
        rc = ensure_transposed_weights(h, s);
        if (rc) return rc;
    }
    __nv_bfloat16* const G = h->G.ptr;
    __nv_bfloat16* const Hr = h->Hr.ptr;
    // deterministic column sums of a row-major [M][N] bf16 matrix into out[N] (fp32):
    // row-block partials, then the blocks added in order; each call site has its own
    // partials region (the side stream's and the caller's sums may overlap in time)
    auto bias_sums = [&](const __nv_bfloat16* X, int N, float* out, float* part, cudaStream_t st) -> int {
        h->launches += 2;
        vlp::vlp_colsum_rows_kernel<<<dim3(static_cast<unsigned>((N / 2 + vlp::CSR_THREADS - 1) / vlp::CSR_THREADS),
                                           static_cast<unsigned>(nb_cs)),
                                      vlp::CSR_THREADS, 0, st>>>(X, M, N, part);
        vlp::vlp_colsum_kernel<<<(N + vlp::CS_COLS - 1) / vlp::CS_COLS, vlp::CS_COLS * vlp::CS_GROUPS, 0, st>>>(
            part, static_cast<int>(nb_cs), N / 2, out, out + N / 2);
        return cudaGetLastError() == cudaSuccess ? VLPROJ_OK : VLPROJ_ERR_CUDA;
    };
    float* const part_b2 = h->part_cs.ptr;
    float* const part_b1 = part_b2 + nb_cs * c.N2;
    float* const part_mid = part_b1 + nb_cs * c.N1;
    rc = upload_plan(h, pl, s);
    if (rc) return rc;
    h->profiled_valid = false;
    for (bool& r : h->stage_ran) r = false;

    // 6. placeholder index, count check, destinations and gather data
    stage_begin(h, 6, s);
    VLP_CUDA(vlp::enqueue_placeholder_index(a->input_ids, n_ids, a->image_token_id, h->counts.ptr, h->pos.ptr, pl.R,
                                            h->status + 1, h->status, nullptr, s, &h->launches));
    if (M == 0) {
        stage_end(h, 6, s);
        rc = zero_outputs(a, c, K1, pl.P, s);
        if (rc) return rc;
        h->profiled_valid = h->profiling;
        return VLPROJ_OK;
    }
    ++h->launches;
    vlp::vlp_geometry_kernel<<<static_cast<unsigned>((M + 255) / 256), 256, 0, s>>>(
        h->dviews.ptr, static_cast<int>(pl.views.size()), static_cast<int>(M), c.k, h->pos.ptr, pl.R,
        vlp::DEST_EMBED, h->gmeta.ptr, h->rowdest.ptr, nullptr, 0, pl.chunk, 0);
    VLP_CUDA(cudaGetLastError());
    stage_end(h, 6, s);

    const float eps = c.ln_eps > 0.f ? c.ln_eps : 1e-5f;
    CUtensorMap tmA{};
    GemmParams p{};

    if (want_recompute) {
        // 7. A, exactly as the forward pass rounds it
        stage_begin(h, 7, s);
        ++h->launches;
        rc = launch_ln_merge(h, a->features, h->dviews.ptr, static_cast<int>(pl.views.size()), static_cast<int>(M), eps,
                             h->A.ptr, s);
        if (rc) return rc;
        stage_end(h, 7, s);

        // 8. every hidden layer recomputed: G_l = GELU'(P_l) and H_l, both row-major (the
        //    weight-gradient GEMMs read H_l as an MN-major operand)
        stage_begin(h, 8, s);
        for (int l = 1; l <= depth - 1; ++l) {
            const bool first = l == 1;
            const __nv_bfloat16* x = first ? h->A.ptr : Hr + (l - 2) * hslab;
            const int K = first ? K1 : c.N1;
            if (encode_bf16_2d(&tmA, x, M, K, vlp::BM)) return VLPROJ_ERR_CUDA;
            p = gemm_params(h, M, c.N1, K);
            p.bias = first ? h->b1 : h->bm[l - 2];
            CUtensorMap tmG{}, tmHr{};
            if (encode_bf16_store(&tmG, G + (l - 1) * hslab, M, c.N1) ||
                encode_bf16_store(&tmHr, Hr + (l - 1) * hslab, M, c.N1))
                return VLPROJ_ERR_CUDA;
            ++h->launches;
            rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_BWD_H>(h, pick_bn(c.N1), h->pairs, tmA,
                                                             first ? h->tmW1 : h->tmWm[l - 2],
                                                             first ? h->tmW1h : h->tmWmh[l - 2], p, s,
                                                             tmG, tmHr);
            if (rc) return rc;
        }
        stage_end(h, 8, s);
    }

    // 9. dY from the placeholder rows of d_out
    stage_begin(h, 9, s);
    ++h->launches;
    transpose_launch(static_cast<const __nv_bfloat16*>(a->d_out), c.N2, n_ids, h->rowdest.ptr, h->status + 1, M,
                     c.N2, h->dY.ptr, nullptr, 0, c.C, 1, 0, s);
    VLP_CUDA(cudaGetLastError());
    stage_end(h, 9, s);

    // Up to about 2^28 hidden activations (M * N1) the top and first layers' weight
    // gradients run on the side stream, beside the dP chain on the caller's stream: the
    // top one needs only stages 7-9, dW1 waits for dP_1, and each persistent GEMM
    // takes the SMs the other leaves free, which fills their partial last waves (measured
    // 1.4-2 % faster on the MoonViT, DeepSeek-ViT and VL2 batches). Larger batches run in
    // sequence: there the two GEMM streams contend for L2 and power (measured 8 % slower
    // on 262,144 tokens).
    const bool overlap = M * c.N1 <= (int64_t(1) << 28);
    cudaStream_t ss = overlap ? h->side : s;
    VLP_CUDA(cudaEventRecord(h->fork, s));
    VLP_CUDA(cudaStreamWaitEvent(ss, h->fork, 0));

    // 11. top layer: dW2 = dY^T H_(depth-1) and db2 (side stream); dY and H are read
    //     where they lie, as MN-major operands
    CUtensorMap tmA2{}, tmB2{}, tmB2h{};
    if (a->d_W2) {
        // N2 need only be a multiple of 32: then dY's 64-column strips come by separate 2D
        // boxes, so the last strip's columns past N2 read as zeros
        const bool strips = c.N2 % 64 != 0;
        const int rc_a = strips ? encode_bf16_2d(&tmA2, h->dY.ptr, M, c.N2, 64)
                                : encode_bf16_mn(&tmA2, h->dY.ptr, M, c.N2, vlp::BM / 64);
        if (rc_a || encode_b_mn(&tmB2, &tmB2h, Hr + (depth - 2) * hslab, M, c.N1, pick_bn(c.N1)))
            return VLPROJ_ERR_CUDA;
        GemmParams q = gemm_params(h, c.N2, c.N1, M);
        q.a_mn = strips ? 2 : 1;
        q.b_mn = 1;
        q.outf = a->d_W2;
        stage_begin(h, 11, ss);
        ++h->launches;
        rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_F32>(h, pick_bn(c.N1), h->pairs, tmA2, tmB2, tmB2h, q, ss);
        if (rc) return rc;
        stage_end(h, 11, ss);
    }
    if (a->d_b2) {
        rc = bias_sums(h->dY.ptr, c.N2, a->d_b2, part_b2, ss);
        if (rc) return rc;
    }

    // 10. the dP chain (caller's stream): dP_l = (dP_(l+1) W_(l+1)) * G_l from the top
    //     down to the lowest layer asked for, with the middle layers' weight gradients
    //     dW_mid = dP^T H and db_mid on the way; dP ping-pongs between two slabs
    int cur = 0;                       // slab holding the latest dP
    if (l_min < depth) {
        stage_begin(h, 10, s);
        for (int l = depth - 1; l >= l_min; --l) {
            // dP_l from dP_(l+1) (dY for the top) through Linear l+1
            const bool top = l == depth - 1;
            const int nxt = top ? 0 : cur ^ 1;
            if (encode_bf16_2d(&tmA, top ? h->dY.ptr : h->dP.ptr + cur * hslab, M, top ? c.N2 : c.N1, vlp::BM))
                return VLPROJ_ERR_CUDA;
            p = gemm_params(h, M, c.N1, top ? c.N2 : c.N1);
            p.aux = G + (l - 1) * hslab;
            CUtensorMap tmP{};
            if (encode_bf16_store(&tmP, h->dP.ptr + nxt * hslab, M, c.N1)) return VLPROJ_ERR_CUDA;
            ++h->launches;
            rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_DGELU>(h, pick_bn(c.N1), h->pairs, tmA,
                                                             top ? h->tmW2t : h->tmWmt[l - 1],
                                                             top ? h->tmW2th : h->tmWmth[l - 1], p, s, tmP);
            if (rc) return rc;
            cur = nxt;
            if (l < 2) continue;
            // Linear l (middle layer l - 2): dW = dP_l^T H_(l-1), db = sum dP_l
            const int i = l - 2;
            if (mid_w(i)) {
                CUtensorMap ta{}, tb{}, tbh{};
                if (encode_bf16_mn(&ta, h->dP.ptr + cur * hslab, M, c.N1, vlp::BM / 64) ||
                    encode_b_mn(&tb, &tbh, Hr + (l - 2) * hslab, M, c.N1, pick_bn(c.N1)))
                    return VLPROJ_ERR_CUDA;
                GemmParams q = gemm_params(h, c.N1, c.N1, M);
                q.a_mn = q.b_mn = 1;
                q.outf = mid_w(i);
                ++h->launches;
                rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_F32>(h, pick_bn(c.N1), h->pairs, ta, tb, tbh, q, s);
                if (rc) return rc;
            }
            if (mid_b(i)) {
                rc = bias_sums(h->dP.ptr + cur * hslab, c.N1, mid_b(i), part_mid, s);
                if (rc) return rc;
            }
        }
        stage_end(h, 10, s);
        VLP_CUDA(cudaEventRecord(h->join2, s));
    }
    // dP_1, when the chain reached it (l_min == 1)
    const __nv_bfloat16* dP1 = h->dP.ptr + cur * hslab;

    // 12. dW1 = dP_1^T A and db1 (side stream, after dP_1): dP_1 and A read where they
    //     lie (MN-major); dW1's columns come out in the kernel's position-outer K order and
    //     go back to the caller's channel-outer order by one small pass
    if (want_l1) VLP_CUDA(cudaStreamWaitEvent(ss, h->join2, 0));
    if (a->d_W1) {
        stage_begin(h, 12, ss);
        const bool unpermute = c.k_order == VLPROJ_ORDER_CHANNEL_OUTER && kk > 1;
        if (encode_bf16_mn(&tmA2, dP1, M, c.N1, vlp::BM / 64) ||
            encode_b_mn(&tmB2, &tmB2h, h->A.ptr, M, K1, pick_bn(K1)))
            return VLPROJ_ERR_CUDA;
        GemmParams q = gemm_params(h, c.N1, K1, M);
        q.a_mn = q.b_mn = 1;
        q.outf = unpermute ? h->dW1p.ptr : a->d_W1;
        ++h->launches;
        rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_F32>(h, pick_bn(K1), h->pairs, tmA2, tmB2, tmB2h, q, ss);
        if (rc) return rc;
        if (unpermute) {
            ++h->launches;
            vlp::vlp_unpermute_cols_kernel<<<dim3(static_cast<unsigned>(c.C / 64), static_cast<unsigned>(c.N1)), 64, 0,
                                             ss>>>(h->dW1p.ptr, a->d_W1, c.C, kk);
            VLP_CUDA(cudaGetLastError());
        }
        stage_end(h, 12, ss);
    }
    if (a->d_b1) {
        rc = bias_sums(dP1, c.N1, a->d_b1, part_b1, ss);
        if (rc) return rc;
    }
    VLP_CUDA(cudaEventRecord(h->join, ss));

    // 13. dA = dP W1p (caller's stream): bf16, position-outer columns, for the LayerNorm
    //     backward; without a LayerNorm the epilogue folds it (fp32) onto the patches as
    //     the feature gradient itself
    if (want_da) {
        if (encode_bf16_2d(&tmA, dP1, M, c.N1, vlp::BM)) return VLPROJ_ERR_CUDA;
        p = gemm_params(h, M, K1, c.N1);
        stage_begin(h, 13, s);
        ++h->launches;
        if (c.has_ln) {
            CUtensorMap tmD{};
            if (encode_bf16_store(&tmD, h->dA.ptr, M, K1)) return VLPROJ_ERR_CUDA;
            p.tma_store = 1;
            rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_BF16>(h, pick_bn(K1), h->pairs, tmA, h->tmW1pt, h->tmW1pth, p,
                                                            s, tmD);
        } else {
            p.outf = a->d_features;
            p.gmeta = h->gmeta.ptr;
            rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_FOLD_F32>(h, pick_bn(K1), h->pairs, tmA, h->tmW1pt, h->tmW1pth,
                                                                p, s);
        }
        if (rc) return rc;
        stage_end(h, 13, s);
    }

    // 14. LayerNorm backward, newline / separator gradients (caller's stream)
    stage_begin(h, 14, s);
    if (want_da && c.has_ln) {
        const int64_t items = M * kk;
        const bool ln_sums = a->d_gamma || a->d_beta;
        const size_t smem = static_cast<size_t>(c.C) * 2 * vlp::LNB_WARPS * 4;
        const bool f32 = c.feat_dtype == VLPROJ_FEAT_F32;
        const int nvec = c.C / 8;
        // one wave of blocks: as many as fit on the SMs at once (their shared-memory
        // accumulators bound it, 3 per SM at C = 1152), so no block starts late with a
        // full share of the rows
#define VLP_LNB(F, V)                                                                                         \
    do {                                                                                                      \
        auto kern = vlp::vlp_ln_backward_kernel<F, V>;                                                        \
        VLP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))); \
        int per_sm = 0;                                                                                       \
        VLP_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem));                   \
        const int nb = static_cast<int>(std::min<int64_t>((items + vlp::LNB_WARPS - 1) / vlp::LNB_WARPS,      \
                                                          std::max(per_sm, 1) * static_cast<int64_t>(h->num_sms))); \
        if (ln_sums && h->part.ensure(static_cast<size_t>(nb) * 2 * c.C)) return VLPROJ_ERR_CUDA;           \
        float* partial = ln_sums ? h->part.ptr : nullptr;                                                     \
        ++h->launches;                                                                                        \
        kern<<<nb, 256, smem, s>>>(a->features, h->gmeta.ptr, static_cast<int>(M), c.k, c.C, h->gamma, eps,   \
                                   h->dA.ptr, a->d_features, partial);                                        \
        VLP_CUDA(cudaGetLastError());                                                                         \
        if (ln_sums) {                                                                                        \
            ++h->launches;                                                                                    \
            vlp::vlp_colsum_kernel<<<(2 * c.C + vlp::CS_COLS - 1) / vlp::CS_COLS, vlp::CS_COLS * vlp::CS_GROUPS, 0, \
                                     s>>>(partial, nb, c.C, a->d_gamma, a->d_beta);                           \
            VLP_CUDA(cudaGetLastError());                                                                     \
        }                                                                                                     \
    } while (0)
        if (nvec <= 64) { if (f32) VLP_LNB(true, 2); else VLP_LNB(false, 2); }
        else if (nvec <= 160) { if (f32) VLP_LNB(true, 5); else VLP_LNB(false, 5); }
        else { if (f32) VLP_LNB(true, 8); else VLP_LNB(false, 8); }
#undef VLP_LNB
    }
    if (!c.has_ln) {
        if (a->d_gamma) VLP_CUDA(cudaMemsetAsync(a->d_gamma, 0, static_cast<size_t>(c.C) * 4, s));
        if (a->d_beta) VLP_CUDA(cudaMemsetAsync(a->d_beta, 0, static_cast<size_t>(c.C) * 4, s));
    }
    if (a->d_newline || a->d_sep) {
        if (tiled && !pl.images.empty()) {
            const int n_img = static_cast<int>(pl.images.size());
            if (h->part_sp.ensure(static_cast<size_t>(n_img) * 2 * c.N2)) return VLPROJ_ERR_CUDA;
            h->launches += 2;
            vlp::vlp_special_grad_kernel<<<dim3((c.N2 + 255) / 256, n_img), 256, 0, s>>>(
                h->dimages.ptr, h->pos.ptr, pl.R, static_cast<const __nv_bfloat16*>(a->d_out), n_ids, c.N2,
                h->status + 1, h->part_sp.ptr);
            vlp::vlp_colsum_kernel<<<(2 * c.N2 + vlp::CS_COLS - 1) / vlp::CS_COLS, vlp::CS_COLS * vlp::CS_GROUPS, 0,
                                     s>>>(h->part_sp.ptr, n_img, c.N2, a->d_newline, a->d_sep);
            VLP_CUDA(cudaGetLastError());
        } else {
            if (a->d_newline) VLP_CUDA(cudaMemsetAsync(a->d_newline, 0, static_cast<size_t>(c.N2) * 4, s));
            if (a->d_sep) VLP_CUDA(cudaMemsetAsync(a->d_sep, 0, static_cast<size_t>(c.N2) * 4, s));
        }
    }
    stage_end(h, 14, s);
    VLP_CUDA(cudaStreamWaitEvent(s, h->join, 0));
    h->profiled_valid = h->profiling;
    return VLPROJ_OK;
}
