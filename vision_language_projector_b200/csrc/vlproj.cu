// C-ABI host library of the vision-to-language projector (declared in vlproj.h).
//
// vlproj_forward enqueues, without any host sync:
//   0. placeholder index   count + compact (ids == image_token_id), count check, and
//                          each GEMM row's destination row; on a side stream forked
//                          from the caller's stream and joined back before step 4
//   1. geometry            per GEMM row: gather data; per im2col chunk: the
//                          coordinates of its first token
//   2. LayerNorm/convert   only with a pre-merge LayerNorm or fp32 features
//   3. GEMM1               im2col merge-gather + tcgen05 MMA + bias + GELU -> H (bf16)
//   4. GEMM2               tcgen05 MMA + bias -> bf16 rows scattered into out_embeds
//   5. special rows        newline / separator rows (2D tiling only)
// Host work per call: argument checks, the closed-form row counts, tensor-map
// encoding, and small descriptor uploads that are skipped while unchanged.
#include "host.cuh"

using namespace vlp_host;

namespace vlp_host {

// Steps 1-3: geometry, LayerNorm/convert, GEMM1. GEMM row m goes to
//   dest_mode DEST_EMBED:   hidden row m (internal H, M rows); pos gives rowdest for GEMM2
//   dest_mode DEST_ROW:     hidden row m; rowdest[m] = the token's assembled row
//   dest_mode DEST_COMPACT: hidden row = merged-token index (caller's buffer, M_real rows)
// dviews: the plan's view table on the device (null = the handle's).
int run_merge_gemm1(vlproj_handle* h, const Plan& pl, const void* features, const int32_t* pos, int dest_mode,
                    __nv_bfloat16* hidden, int64_t hidden_rows, cudaStream_t s, const ViewDesc* dviews) {
    if (!dviews) dviews = h->dviews.ptr;
    const vlproj_config& c = h->cfg;
    const int M = static_cast<int>(pl.M);
    if (M == 0) return VLPROJ_OK;
    const bool im2col = pl.im2col;
    const int nch_tile = vlp::BM / pl.chunk;
    // chunk entries for every 128-row slice of every (pair) tile, so round to 256 rows
    const int n_chunks = im2col ? ((M + 2 * vlp::BM - 1) / (2 * vlp::BM)) * 2 * nch_tile : 0;
    // gather metadata only for GEMM1's cp.async gather (the merged-LayerNorm pass finds its
    // source rows in the view table, the box and im2col modes need none)
    const bool cpasync = !im2col && !pl.box5 && !pl.merged_ln && !pl.fused;   // includes the thread gather
    if (h->rowdest.ensure(M)) return VLPROJ_ERR_CUDA;
    if (cpasync && h->gmeta.ensure(M)) return VLPROJ_ERR_CUDA;
    if (im2col && h->chunks.ensure(std::max(n_chunks, 1))) return VLPROJ_ERR_CUDA;

    // the geometry pass only when something below reads its output (a forward with the
    // merged LayerNorm or the box gather and no row table skips it)
    if (cpasync || im2col || dest_mode != vlp::DEST_NONE) {
        stage_begin(h, 1, s);
        ++h->launches;
        const int geo_threads = std::max(M, n_chunks);
        vlp::vlp_geometry_kernel<<<(geo_threads + 255) / 256, 256, 0, s>>>(
            dviews, static_cast<int>(pl.views.size()), M, c.k, pos, pl.R, dest_mode,
            cpasync ? h->gmeta.ptr : nullptr, h->rowdest.ptr, im2col ? h->chunks.ptr : nullptr, n_chunks, pl.chunk,
            pl.uniform ? 1 : 0);
        VLP_CUDA(cudaGetLastError());
        stage_end(h, 1, s);
    }

    const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(features);
    // A_TGATHER_LN: rows of the statistics table, whole 256-row tiles
    const int64_t stats_ld = (static_cast<int64_t>(M) + 255) / 256 * 256;
    if (pl.tgather_ln) {
        stage_begin(h, 2, s);
        ++h->launches;
        const int kk = c.k * c.k;
        if (h->lnstats.ensure(static_cast<size_t>(stats_ld) * kk)) return VLPROJ_ERR_CUDA;
        const float eps = c.ln_eps > 0.f ? c.ln_eps : 1e-5f;
        const int64_t items = stats_ld * kk;
        vlp::vlp_ln_stats_kernel<false><<<static_cast<unsigned>((items + 7) / 8), 256, 0, s>>>(
            features, dviews, static_cast<int>(pl.views.size()), M, stats_ld, c.k, c.C, eps, h->lnstats.ptr);
        VLP_CUDA(cudaGetLastError());
        stage_end(h, 2, s);
    } else if (pl.merged_ln) {
        stage_begin(h, 2, s);
        ++h->launches;
        if (h->A.ensure(static_cast<size_t>(M) * h->K1)) return VLPROJ_ERR_CUDA;
        const float eps = c.ln_eps > 0.f ? c.ln_eps : 1e-5f;
        int rc = launch_ln_merge(h, features, dviews, static_cast<int>(pl.views.size()), M, eps, h->A.ptr, s);
        if (rc) return rc;
        stage_end(h, 2, s);
    } else if ((c.has_ln || c.feat_dtype == VLPROJ_FEAT_F32) && !pl.tgather_ln && !pl.fused) {
        stage_begin(h, 2, s);
        ++h->launches;
        if (h->Xn.ensure(static_cast<size_t>(pl.P) * c.C)) return VLPROJ_ERR_CUDA;
        const unsigned blocks = static_cast<unsigned>((pl.P + 7) / 8);
        const float eps = c.ln_eps > 0.f ? c.ln_eps : 1e-5f;
        if (c.feat_dtype == VLPROJ_FEAT_F32)
            vlp::vlp_layernorm_kernel<true><<<blocks, 256, 0, s>>>(features, pl.P, c.C, h->gamma, h->beta, eps,
                                                                   c.has_ln, h->Xn.ptr);
        else
            vlp::vlp_layernorm_kernel<false><<<blocks, 256, 0, s>>>(features, pl.P, c.C, h->gamma, h->beta, eps,
                                                                    c.has_ln, h->Xn.ptr);
        VLP_CUDA(cudaGetLastError());
        stage_end(h, 2, s);
        src = h->Xn.ptr;
    }

    GemmParams p{};
    p.M = M;
    p.N = c.N1;
    p.K = h->K1;
    p.bias = h->b1;
    p.C = c.C;
    p.k = c.k;
    p.out = hidden;
    p.rowdest = dest_mode == vlp::DEST_COMPACT ? h->rowdest.ptr : nullptr;
    p.out_rows = hidden_rows;
    // GEMM row m is hidden row m unless rows are remapped: then rows leave by TMA store
    CUtensorMap tmC{};
    p.tma_store = p.rowdest == nullptr ? 1 : 0;
    if (p.tma_store && encode_bf16_store(&tmC, hidden, static_cast<uint64_t>(hidden_rows), c.N1))
        return VLPROJ_ERR_CUDA;
    p.fwd_status = nullptr;
    p.err = h->status;
    p.wait_ns = h->wait_ns;
    p.l2_budget = h->l2_budget;

    CUtensorMap tmA{};
    std::memset(&tmA, 0, sizeof(tmA));
    if (pl.merged_ln) {
        if (encode_bf16_2d(&tmA, h->A.ptr, static_cast<uint64_t>(M), static_cast<uint64_t>(h->K1), vlp::BM))
            return VLPROJ_ERR_CUDA;
    } else if (pl.fused) {
        // A written by GEMM1's producer warps, read back by its TMA tiles; counters zeroed
        const int kk = c.k * c.k;
        const int m_blocks = (M + vlp::FUSED_BLOCK - 1) / vlp::FUSED_BLOCK;
        const size_t words = 2 + static_cast<size_t>(m_blocks) * kk;
        if (h->A.ensure(static_cast<size_t>(M) * h->K1) || h->fwork.ensure(words)) return VLPROJ_ERR_CUDA;
        VLP_CUDA(cudaMemsetAsync(h->fwork.ptr, 0, words * sizeof(uint32_t), s));
        if (encode_bf16_2d(&tmA, h->A.ptr, static_cast<uint64_t>(M), static_cast<uint64_t>(h->K1), vlp::BM))
            return VLPROJ_ERR_CUDA;
        p.views = dviews;
        p.n_views = static_cast<int>(pl.views.size());
        p.feat = features;
        p.feat_f32 = c.feat_dtype == VLPROJ_FEAT_F32 ? 1 : 0;
        p.has_ln = c.has_ln ? 1 : 0;
        p.ln_eps = c.ln_eps > 0.f ? c.ln_eps : 1e-5f;
        p.ln_gamma = h->gamma;
        p.ln_beta = h->beta;
        p.a_out = h->A.ptr;
        p.work = reinterpret_cast<unsigned long long*>(h->fwork.ptr);
        p.ready = h->fwork.ptr + 2;
        p.m_blocks = m_blocks;
    } else if (pl.box5) {
        const ViewDesc& V = pl.views[0];
        if (encode_box5(&tmA, src, c.C, V.h, V.w, static_cast<int>(pl.views.size()), c.k)) return VLPROJ_ERR_CUDA;
        p.box_rows = vlp::BM / V.wp;
    } else if (im2col) {
        p.chunks = h->chunks.ptr;
        p.chunk = pl.chunk;
        if (pl.uniform) {
            const ViewDesc& V = pl.views[0];
            if (encode_im2col(&tmA, src, c.C, V.h, V.w, static_cast<int>(pl.views.size()), c.k, pl.chunk))
                return VLPROJ_ERR_CUDA;
            p.gmaps = nullptr;
            p.n_gmaps = 0;
        } else {
            h->host_maps.resize(pl.views.size());
            for (size_t v = 0; v < pl.views.size(); ++v) {
                const ViewDesc& V = pl.views[v];
                if (encode_im2col(&h->host_maps[v], src + V.patch_start * c.C, c.C, V.h, V.w, 1, c.k, pl.chunk))
                    return VLPROJ_ERR_CUDA;
            }
            if (h->dmaps.ptr == nullptr || h->dmaps.cap < pl.views.size()) h->up_maps.invalidate();
            if (h->dmaps.ensure(pl.views.size())) return VLPROJ_ERR_CUDA;
            int rc = h->up_maps.put(h->dmaps.ptr, h->host_maps.data(), pl.views.size() * sizeof(CUtensorMap), s);
            if (rc) return rc;
            p.gmaps = h->dmaps.ptr;
            p.n_gmaps = static_cast<int>(pl.views.size());
        }
    } else {
        p.gsrc = src;
        p.gmeta = h->gmeta.ptr;
        if (pl.tgather_ln) {
            p.ln_stats = h->lnstats.ptr;
            p.stats_ld = stats_ld;
            p.ln_gamma = h->gamma;
            p.ln_beta = h->beta;
        }
    }

    stage_begin(h, 3, s);
    ++h->launches;
    int rc;
    if (pl.fused)
        rc = launch_gemm_bn<vlp::A_FUSED, vlp::EPI_GELU>(h, pick_bn(c.N1), h->pairs, tmA, h->tmW1, h->tmW1h, p,
                                                         s, tmC);
    else if (pl.tgather_ln)
        rc = launch_gemm_bn<vlp::A_TGATHER_LN, vlp::EPI_GELU>(h, pick_bn(c.N1), h->pairs, tmA, h->tmW1, h->tmW1h, p,
                                                              s, tmC);
    else if (pl.tgather)
        rc = launch_gemm_bn<vlp::A_TGATHER, vlp::EPI_GELU>(h, pick_bn(c.N1), h->pairs, tmA, h->tmW1, h->tmW1h, p,
                                                           s, tmC);
    else if (pl.merged_ln)
        rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_GELU>(h, pick_bn(c.N1), h->pairs, tmA, h->tmW1, h->tmW1h, p,
                                                        s, tmC);
    else if (pl.box5)
        rc = launch_gemm_bn<vlp::A_BOX5, vlp::EPI_GELU>(h, pick_bn(c.N1), h->pairs, tmA, h->tmW1, h->tmW1h, p,
                                                        s, tmC);
    else if (im2col)      // 256 x 512 pair tiles where N1 allows: each im2col load feeds two MMAs
        rc = launch_gemm_bn<vlp::A_IM2COL, vlp::EPI_GELU>(h, c.N1 % 512 == 0 ? 512 : pick_bn(c.N1), h->pairs, tmA,
                                                          h->tmW1, h->tmW1h, p, s, tmC);
    else
        rc = launch_gemm_bn<vlp::A_CPASYNC, vlp::EPI_GELU>(h, pick_bn(c.N1), false, tmA, h->tmW1, h->tmW1h, p,
                                                           s, tmC);
    if (rc) return rc;
    stage_end(h, 3, s);
    return VLPROJ_OK;
}

// Middle layers (depth > 2): H <- bf16(GELU(H Wm^T + bm)), ping-pong between H and H2.
// *hlast: the buffer holding the last hidden activation.
int run_middle_layers(vlproj_handle* h, const Plan& pl, cudaStream_t s, const __nv_bfloat16** hlast) {
    const vlproj_config& c = h->cfg;
    bool last_in_h2 = false;
    for (int layer = 0; layer + 2 < c.depth; ++layer) {
        DevBuf<__nv_bfloat16>& src = last_in_h2 ? h->H2 : h->H;
        DevBuf<__nv_bfloat16>& dst = last_in_h2 ? h->H : h->H2;
        CUtensorMap tin{};
        if (encode_bf16_2d(&tin, src.ptr, pl.M, c.N1, vlp::BM)) return VLPROJ_ERR_CUDA;
        GemmParams q{};
        q.M = static_cast<int>(pl.M);
        q.N = c.N1;
        q.K = c.N1;
        q.bias = h->bm[layer];
        q.C = c.C;
        q.k = c.k;
        q.out = dst.ptr;
        q.out_rows = pl.M;
        q.err = h->status;
        q.wait_ns = h->wait_ns;
        CUtensorMap tout{};
        q.tma_store = 1;
        if (encode_bf16_store(&tout, dst.ptr, pl.M, c.N1)) return VLPROJ_ERR_CUDA;
        ++h->launches;
        int rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_GELU>(h, pick_bn(c.N1), h->pairs, tin, h->tmWm[layer],
                                                            h->tmWmh[layer], q, s, tout);
        if (rc) return rc;
        last_in_h2 = !last_in_h2;
    }
    *hlast = last_in_h2 ? h->H2.ptr : h->H.ptr;
    return VLPROJ_OK;
}

}  // namespace vlp_host

extern "C" {

const char* vlproj_strerror(int code) {
    switch (code) {
        case VLPROJ_OK: return "ok";
        case VLPROJ_ERR_INVALID_ARG: return "invalid argument";
        case VLPROJ_ERR_UNSUPPORTED: return "unsupported projector configuration";
        case VLPROJ_ERR_CUDA: return "CUDA error";
        case VLPROJ_ERR_TOKEN_COUNT: return "placeholder count does not match the image rows";
        case VLPROJ_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
        default: return "unknown status";
    }
}

const char* vlproj_version(void) { return "vlproj 0.2 sm_100a"; }

int64_t vlproj_image_rows(const vlproj_config* cfg, const int32_t* grid_hw, const int32_t* spatial_crop,
                          int32_t n_images, int64_t* rows_out) {
    int rc = validate_config(cfg);
    if (rc) return rc;
    Plan pl;
    rc = build_plan(*cfg, grid_hw, spatial_crop, n_images, false, VLPROJ_GATHER_CPASYNC, &pl);
    if (rc) return rc;
    if (rows_out) {
        // rows of image i = (row_base of the next image) - (its own)
        std::vector<int64_t> base;
        if (cfg->tile_tag == VLPROJ_TILE_2D) {
            for (auto& im : pl.images) base.push_back(im.row_base);
        } else {
            for (auto& v : pl.views) base.push_back(v.row_base);
        }
        base.push_back(pl.R);
        for (int32_t i = 0; i < n_images; ++i) rows_out[i] = base[i + 1] - base[i];
    }
    return pl.R;
}

int64_t vlproj_plan_tiles(const int32_t* image_wh, int32_t n_images, const int32_t* candidates, int32_t n_candidates,
                          int32_t image_size, int32_t patch_size, int32_t downsample, int32_t* spatial_crop_out,
                          int64_t* rows_out) {
    if (n_images < 0 || (n_images > 0 && (!image_wh || !spatial_crop_out)) || image_size <= 0 || patch_size <= 0 ||
        downsample <= 0 || patch_size > image_size)
        return VLPROJ_ERR_INVALID_ARG;
    const bool crop = n_images <= 2;
    if (crop && n_images > 0 && (n_candidates <= 0 || !candidates)) return VLPROJ_ERR_INVALID_ARG;
    const int64_t g = image_size / patch_size;
    const int64_t hp = (g + downsample - 1) / downsample;
    int64_t views = 0;
    for (int32_t i = 0; i < n_images; ++i) {
        const int64_t w0 = image_wh[2 * i], h0 = image_wh[2 * i + 1];
        if (w0 <= 0 || h0 <= 0) return VLPROJ_ERR_INVALID_ARG;
        int64_t W = image_size, H = image_size;
        if (crop) {
            int64_t best_eff = -1, best_waste = 0;
            for (int32_t c = 0; c < n_candidates; ++c) {
                const int64_t cw = candidates[2 * c], ch = candidates[2 * c + 1];
                if (cw <= 0 || ch <= 0 || cw % image_size || ch % image_size) return VLPROJ_ERR_INVALID_ARG;
                const double scale = std::min(static_cast<double>(cw) / static_cast<double>(w0),
                                              static_cast<double>(ch) / static_cast<double>(h0));
                const int64_t fw = static_cast<int64_t>(std::floor(static_cast<double>(w0) * scale));
                const int64_t fh = static_cast<int64_t>(std::floor(static_cast<double>(h0) * scale));
                const int64_t eff = std::min(fw * fh, w0 * h0);
                const int64_t waste = cw * ch - eff;
                if (eff > best_eff || (eff == best_eff && waste < best_waste)) {
                    best_eff = eff;
                    best_waste = waste;
                    W = cw;
                    H = ch;
                }
            }
        }
        const int64_t tw = W / image_size, th = H / image_size;
        spatial_crop_out[2 * i] = static_cast<int32_t>(tw);
        spatial_crop_out[2 * i + 1] = static_cast<int32_t>(th);
        if (rows_out) rows_out[i] = hp * (hp + 1) + 1 + (th * hp) * (tw * hp + 1);
        views += 1 + tw * th;
    }
    return views;
}

int vlproj_create(const vlproj_config* cfg, vlproj_handle** out) {
    if (!out) return VLPROJ_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = validate_config(cfg);
    if (rc) return rc;
    if (!cfg->W1 || !cfg->W2 || (cfg->has_ln && (!cfg->ln_gamma || !cfg->ln_beta))) return VLPROJ_ERR_INVALID_ARG;
    if (cfg->depth > 2) {
        if (!cfg->W_mid) return VLPROJ_ERR_INVALID_ARG;
        for (int i = 0; i < cfg->depth - 2; ++i)
            if (!cfg->W_mid[i]) return VLPROJ_ERR_INVALID_ARG;
    }
    if (!driver().tiled || !driver().im2col) return VLPROJ_ERR_CUDA;

    vlproj_handle* h = new vlproj_handle();
    h->cfg = *cfg;
    h->K1 = cfg->k * cfg->k * cfg->C;
    auto fail = [&](int code) {
        vlproj_destroy(h);
        return code;
    };
    if (cudaGetDevice(&h->device) != cudaSuccess) return fail(VLPROJ_ERR_CUDA);
    if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess)
        return fail(VLPROJ_ERR_CUDA);
    const size_t n1 = static_cast<size_t>(cfg->N1), n2 = static_cast<size_t>(cfg->N2), C = static_cast<size_t>(cfg->C);
    if (cudaMalloc(&h->W1p, n1 * h->K1 * 2) || cudaMalloc(&h->W2, n2 * n1 * 2) || cudaMalloc(&h->b1, n1 * 4) ||
        cudaMalloc(&h->b2, n2 * 4) || cudaMalloc(&h->gamma, C * 4) || cudaMalloc(&h->beta, C * 4) ||
        cudaMalloc(&h->status, 2 * sizeof(int)) || cudaMalloc(&h->tqueue, 2 * kTileQueues * sizeof(int)) ||
        cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) ||
        cudaEventCreateWithFlags(&h->fork, cudaEventDisableTiming) ||
        cudaEventCreateWithFlags(&h->join, cudaEventDisableTiming) ||
        cudaEventCreateWithFlags(&h->join2, cudaEventDisableTiming))
        return fail(VLPROJ_ERR_CUDA);
    cudaStream_t s = nullptr;
    vlp::vlp_permute_w1_kernel<<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(cfg->W1), h->W1p,
                                                    cfg->N1, cfg->C, cfg->k * cfg->k,
                                                    cfg->k_order == VLPROJ_ORDER_POSITION_OUTER);
    if (cudaGetLastError() != cudaSuccess) return fail(VLPROJ_ERR_CUDA);
    ++h->launches;
    if (cudaMemcpy(h->W2, cfg->W2, n2 * n1 * 2, cudaMemcpyDeviceToDevice)) return fail(VLPROJ_ERR_CUDA);
    if (cfg->b1 ? cudaMemcpy(h->b1, cfg->b1, n1 * 4, cudaMemcpyDeviceToDevice) : cudaMemset(h->b1, 0, n1 * 4))
        return fail(VLPROJ_ERR_CUDA);
    if (cfg->b2 ? cudaMemcpy(h->b2, cfg->b2, n2 * 4, cudaMemcpyDeviceToDevice) : cudaMemset(h->b2, 0, n2 * 4))
        return fail(VLPROJ_ERR_CUDA);
    if (cfg->has_ln) {
        if (cudaMemcpy(h->gamma, cfg->ln_gamma, C * 4, cudaMemcpyDeviceToDevice) ||
            cudaMemcpy(h->beta, cfg->ln_beta, C * 4, cudaMemcpyDeviceToDevice))
            return fail(VLPROJ_ERR_CUDA);
    } else if (cudaMemset(h->gamma, 0, C * 4) || cudaMemset(h->beta, 0, C * 4)) {
        return fail(VLPROJ_ERR_CUDA);
    }
    if (cudaMemset(h->status, 0, 2 * sizeof(int)) || cudaMemset(h->tqueue, 0, 2 * kTileQueues * sizeof(int)))
        return fail(VLPROJ_ERR_CUDA);
    if (cudaDeviceSynchronize()) return fail(VLPROJ_ERR_CUDA);
    for (int i = 0; i < cfg->depth - 2; ++i) {
        __nv_bfloat16* w = nullptr;
        float* b = nullptr;
        if (cudaMalloc(&w, n1 * n1 * 2) || cudaMalloc(&b, n1 * 4)) {
            if (w) cudaFree(w);
            return fail(VLPROJ_ERR_CUDA);
        }
        h->Wm.push_back(w);
        h->bm.push_back(b);
        const float* bsrc = cfg->b_mid ? cfg->b_mid[i] : nullptr;
        if (cudaMemcpy(w, cfg->W_mid[i], n1 * n1 * 2, cudaMemcpyDeviceToDevice) ||
            (bsrc ? cudaMemcpy(b, bsrc, n1 * 4, cudaMemcpyDeviceToDevice) : cudaMemset(b, 0, n1 * 4)))
            return fail(VLPROJ_ERR_CUDA);
        CUtensorMap full{}, half{};
        if (encode_bf16_2d(&full, w, n1, n1, pick_bn(cfg->N1)) || encode_bf16_2d(&half, w, n1, n1, 128))
            return fail(VLPROJ_ERR_CUDA);
        h->tmWm.push_back(full);
        h->tmWmh.push_back(half);
    }
    if (cudaDeviceSynchronize()) return fail(VLPROJ_ERR_CUDA);
    h->cfg.W_mid = nullptr;       // the caller's arrays are not kept
    h->cfg.b_mid = nullptr;
    if (encode_bf16_2d(&h->tmW1, h->W1p, n1, h->K1, pick_bn(cfg->N1)) ||
        encode_bf16_2d(&h->tmW2, h->W2, n2, n1, pick_bn(cfg->N2)) ||
        encode_bf16_2d(&h->tmW1h, h->W1p, n1, h->K1, 128) || encode_bf16_2d(&h->tmW2h, h->W2, n2, n1, 128))
        return fail(VLPROJ_ERR_CUDA);
    *out = h;
    return VLPROJ_OK;
}

void vlproj_destroy(vlproj_handle* h) {
    if (!h) return;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    cudaFree(h->W1p);
    cudaFree(h->W2);
    cudaFree(h->b1);
    cudaFree(h->b2);
    cudaFree(h->gamma);
    cudaFree(h->beta);
    cudaFree(h->status);
    cudaFree(h->tqueue);
    h->H.release();
    h->H2.release();
    cudaFree(h->W2t);
    cudaFree(h->W1pt);
    for (auto* w : h->Wmt) cudaFree(w);
    for (auto* b : {&h->G, &h->Hr, &h->dY, &h->dP}) b->release();
    h->dW1p.release();
    h->part_cs.release();
    h->dA.release();
    h->part.release();
    h->part_sp.release();
    for (int i = 0; i < 2; ++i) {
        h->stage_feat[i].release();
        h->stage_rows[i].release();
        if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
        if (h->ev_done[i]) cudaEventDestroy(h->ev_done[i]);
        if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    }
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
    for (auto* w : h->Wm) cudaFree(w);
    for (auto* b : h->bm) cudaFree(b);
    h->Xn.release();
    h->A.release();
    h->pos.release();
    h->rowdest.release();
    h->counts.release();
    h->gmeta.release();
    h->lnstats.release();
    h->fwork.release();
    h->chunks.release();
    h->dviews.release();
    h->dimages.release();
    h->dmaps.release();
    h->up_views.release();
    h->up_images.release();
    h->up_maps.release();
    for (auto& e : h->ev_begin)
        if (e) cudaEventDestroy(e);
    for (auto& e : h->ev_end)
        if (e) cudaEventDestroy(e);
    if (h->fork) cudaEventDestroy(h->fork);
    if (h->join) cudaEventDestroy(h->join);
    if (h->join2) cudaEventDestroy(h->join2);
    if (h->side) cudaStreamDestroy(h->side);
    cudaSetDevice(cur);
    delete h;
}

int vlproj_set_wait_limit(vlproj_handle* h, uint64_t ns) {
    if (!h) return VLPROJ_ERR_INVALID_ARG;
    h->wait_ns = ns ? ns : kDefaultWaitNs;
    return VLPROJ_OK;
}

int vlproj_set_raster_budget(vlproj_handle* h, int64_t bytes) {
    if (!h || bytes < 0) return VLPROJ_ERR_INVALID_ARG;
    h->l2_budget = bytes;
    return VLPROJ_OK;
}

int vlproj_set_tile_order(vlproj_handle* h, int order) {
    if (!h || order < VLPROJ_TILE_ORDER_STATIC || order > VLPROJ_TILE_ORDER_DYNAMIC) return VLPROJ_ERR_INVALID_ARG;
    h->tile_order = order;
    return VLPROJ_OK;
}

int vlproj_set_tile_pairs(vlproj_handle* h, int enable) {
    if (!h) return VLPROJ_ERR_INVALID_ARG;
    h->pairs = enable != 0;
    return VLPROJ_OK;
}

int vlproj_set_gather_mode(vlproj_handle* h, int mode) {
    if (!h || mode < VLPROJ_GATHER_IM2COL || mode > VLPROJ_GATHER_MERGED)
        return VLPROJ_ERR_INVALID_ARG;
    h->gather_mode = mode;
    return VLPROJ_OK;
}

int vlproj_status(vlproj_handle* h, void* stream) {
    if (!h) return VLPROJ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    VLP_CUDA(cudaStreamSynchronize(s));
    int st = 0;
    VLP_CUDA(cudaMemcpy(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost));
    VLP_CUDA(cudaMemset(h->status, 0, sizeof(int)));
    return st;
}

int vlproj_hidden(vlproj_handle* h, const void* features, const int32_t* grid_hw, int32_t n_views, void* hidden,
                  void* stream) {
    if (!h || n_views < 0 || (n_views > 0 && (!features || !grid_hw || !hidden))) return VLPROJ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(features) % 16 || reinterpret_cast<uintptr_t>(hidden) % 16)
        return VLPROJ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Plan pl;
    int rc = build_plan(h->cfg, grid_hw, nullptr, n_views, true, h->gather_mode, &pl);
    if (rc) return rc;
    if (pl.M == 0) return VLPROJ_OK;
    h->profiled_valid = false;
    rc = upload_plan(h, pl, s);
    if (rc) return rc;
    return run_merge_gemm1(h, pl, features, nullptr, vlp::DEST_COMPACT, static_cast<__nv_bfloat16*>(hidden),
                           pl.M_real, s, nullptr);
}

int vlproj_forward(vlproj_handle* h, const void* features, const int32_t* grid_hw, const int32_t* spatial_crop,
                   int32_t n_images, const int64_t* input_ids, int64_t n_ids, int64_t image_token_id,
                   const void* newline, const void* sep, void* out_embeds, void* stream) {
    vlproj_forward_args a{};
    a.features = features;
    a.grid_hw = grid_hw;
    a.spatial_crop = spatial_crop;
    a.n_images = n_images;
    a.input_ids = input_ids;
    a.n_ids = n_ids;
    a.image_token_id = image_token_id;
    a.newline = newline;
    a.sep = sep;
    a.out_embeds = out_embeds;
    return vlproj_forward_ex(h, &a, stream);
}

int vlproj_forward_ex(vlproj_handle* h, const vlproj_forward_args* args, void* stream) {
    if (!h || !args) return VLPROJ_ERR_INVALID_ARG;
    const void* features = args->features;
    const int32_t* grid_hw = args->grid_hw;
    const int32_t* spatial_crop = args->spatial_crop;
    const int32_t n_images = args->n_images;
    const int64_t* input_ids = args->input_ids;
    const int64_t n_ids = args->n_ids;
    const int64_t image_token_id = args->image_token_id;
    const void* newline = args->newline;
    const void* sep = args->sep;
    void* out_embeds = args->out_embeds;
    const vlproj_config& c = h->cfg;
    if (n_ids < 0 || n_ids >= (int64_t(1) << 31)) return VLPROJ_ERR_INVALID_ARG;
    if (n_ids > 0 && (!input_ids || !out_embeds)) return VLPROJ_ERR_INVALID_ARG;
    if (n_images > 0 && !features) return VLPROJ_ERR_INVALID_ARG;
    const bool tiled = c.tile_tag == VLPROJ_TILE_2D;
    if (tiled && n_images > 0 && (!newline || !sep)) return VLPROJ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(out_embeds) % 16 || reinterpret_cast<uintptr_t>(features) % 16 ||
        (tiled && (reinterpret_cast<uintptr_t>(newline) % 16 || reinterpret_cast<uintptr_t>(sep) % 16)))
        return VLPROJ_ERR_INVALID_ARG;
    if (args->embed_table && (args->vocab <= 0 || reinterpret_cast<uintptr_t>(args->embed_table) % 16))
        return VLPROJ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Plan pl;
    int rc = build_plan(c, grid_hw, spatial_crop, n_images, false, h->gather_mode, &pl);
    if (rc) return rc;
    if (args->rows_out && (args->rows_out_cap < pl.R || reinterpret_cast<uintptr_t>(args->rows_out) % 16))
        return VLPROJ_ERR_INVALID_ARG;
    const bool lookup = args->embed_table != nullptr && n_ids > 0;

    // 0. placeholder index (and each GEMM row's destination), on the side stream so it
    //    overlaps the geometry / LayerNorm / GEMM1 chain on the caller's stream
    const int nblocks = vlp::scan_blocks(n_ids);
    if (h->counts.ensure(nblocks + 1) || h->pos.ensure(std::max<int64_t>(pl.R, 1))) return VLPROJ_ERR_CUDA;
    if (pl.M > 0 && h->rowdest.ensure(pl.M)) return VLPROJ_ERR_CUDA;
    if (pl.M > 0 && h->H.ensure(static_cast<size_t>(pl.M) * c.N1)) return VLPROJ_ERR_CUDA;
    if (pl.M > 0 && c.depth > 2 && h->H2.ensure(static_cast<size_t>(pl.M) * c.N1)) return VLPROJ_ERR_CUDA;
    rc = upload_plan(h, pl, s);
    if (rc) return rc;
    h->profiled_valid = false;
    for (bool& r : h->stage_ran) r = false;
    cudaStream_t si = (pl.M > 0 || lookup) ? h->side : s;
    if (si != s) {
        VLP_CUDA(cudaEventRecord(h->fork, s));
        VLP_CUDA(cudaStreamWaitEvent(si, h->fork, 0));
    }
    // a launch error on the side stream still leaves the caller's stream ordered after it
    auto fail_side = [&](int code) {
        if (si != s && cudaEventRecord(h->join, si) == cudaSuccess) cudaStreamWaitEvent(s, h->join, 0);
        return code;
    };
    stage_begin(h, 0, si);
    if (vlp::enqueue_placeholder_index(input_ids, n_ids, image_token_id, h->counts.ptr, h->pos.ptr, pl.R,
                                       h->status + 1, h->status, nullptr, si, &h->launches) != cudaSuccess)
        return fail_side(VLPROJ_ERR_CUDA);
    if (pl.M > 0) {
        ++h->launches;
        const int M = static_cast<int>(pl.M);
        vlp::vlp_geometry_kernel<<<(M + 255) / 256, 256, 0, si>>>(h->dviews.ptr, static_cast<int>(pl.views.size()),
                                                                  M, c.k, h->pos.ptr, pl.R, vlp::DEST_EMBED, nullptr,
                                                                  h->rowdest.ptr, nullptr, 0, pl.chunk, 0);
        if (cudaGetLastError() != cudaSuccess) return fail_side(VLPROJ_ERR_CUDA);
    }
    stage_end(h, 0, si);
    if (si != s) VLP_CUDA(cudaEventRecord(h->join, si));
    if (lookup) {
        // token-embedding rows: independent of the projector, overlaps the GEMMs
        ++h->launches;
        vlp::vlp_embed_lookup_kernel<<<static_cast<unsigned>((n_ids + 7) / 8), 256, 0, si>>>(
            input_ids, n_ids, image_token_id, static_cast<const __nv_bfloat16*>(args->embed_table), args->vocab,
            static_cast<__nv_bfloat16*>(out_embeds), c.N2, h->status);
        if (cudaGetLastError() != cudaSuccess) return fail_side(VLPROJ_ERR_CUDA);
        VLP_CUDA(cudaEventRecord(h->join2, si));
    }
    if (pl.M == 0) {
        if (si != s) VLP_CUDA(cudaStreamWaitEvent(s, lookup ? h->join2 : h->join, 0));
        h->profiled_valid = h->profiling;
        return VLPROJ_OK;
    }

    // An error past this point still orders the caller's stream after the side stream's
    // work (the index and lookup kernels write pos and out_embeds), as a success does.
    auto fail_joined = [&](int code) {
        if (si != s) {
            cudaStreamWaitEvent(s, h->join, 0);
            if (lookup) cudaStreamWaitEvent(s, h->join2, 0);
        }
        return code;
    };
    // 1-3. geometry, LayerNorm, GEMM1 -> H
    rc = run_merge_gemm1(h, pl, features, nullptr, vlp::DEST_NONE, h->H.ptr, pl.M, s, nullptr);
    if (rc) return fail_joined(rc);
    // middle layers (depth > 2)
    const __nv_bfloat16* hlast = nullptr;
    rc = run_middle_layers(h, pl, s, &hlast);
    if (rc) return fail_joined(rc);
    if (cudaStreamWaitEvent(s, h->join, 0) != cudaSuccess) return fail_joined(VLPROJ_ERR_CUDA);

    // 4. GEMM2 + scatter (from the last hidden activation)
    if (h->tmH_ptr != hlast || h->tmH_rows != pl.M) {
        if (encode_bf16_2d(&h->tmH, hlast, pl.M, c.N1, vlp::BM)) return fail_joined(VLPROJ_ERR_CUDA);
        h->tmH_ptr = hlast;
        h->tmH_rows = pl.M;
    }
    GemmParams p{};
    p.M = static_cast<int>(pl.M);
    p.N = c.N2;
    p.K = c.N1;
    p.bias = h->b2;
    p.C = c.C;
    p.k = c.k;
    p.out = static_cast<__nv_bfloat16*>(out_embeds);
    p.rowdest = h->rowdest.ptr;
    p.out_rows = n_ids;
    p.fwd_status = h->status + 1;
    p.err = h->status;
    p.wait_ns = h->wait_ns;
    p.l2_budget = h->l2_budget;
    stage_begin(h, 4, s);
    ++h->launches;
    rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_SCATTER>(h, pick_bn(c.N2), h->pairs, h->tmH, h->tmW2, h->tmW2h, p,
                                                       s);
    if (rc) return fail_joined(rc);
    stage_end(h, 4, s);

    // 5. newline / separator rows
    if (tiled && !pl.images.empty()) {
        stage_begin(h, 5, s);
        ++h->launches;
        dim3 grid(pl.max_special, static_cast<unsigned>(pl.images.size()));
        vlp::vlp_special_rows_kernel<<<grid, 128, 0, s>>>(h->dimages.ptr, h->pos.ptr, pl.R,
                                                          static_cast<const __nv_bfloat16*>(newline),
                                                          static_cast<const __nv_bfloat16*>(sep),
                                                          static_cast<__nv_bfloat16*>(out_embeds), n_ids, c.N2,
                                                          h->status + 1);
        if (cudaGetLastError() != cudaSuccess) return fail_joined(VLPROJ_ERR_CUDA);
        stage_end(h, 5, s);
    }
    if (args->rows_out && pl.R > 0) {
        ++h->launches;
        vlp::vlp_gather_rows_kernel<<<static_cast<unsigned>((pl.R + 7) / 8), 256, 0, s>>>(
            h->pos.ptr, pl.R, static_cast<const __nv_bfloat16*>(out_embeds), n_ids, c.N2,
            static_cast<__nv_bfloat16*>(args->rows_out), h->status + 1);
        if (cudaGetLastError() != cudaSuccess) return fail_joined(VLPROJ_ERR_CUDA);
    }
    if (lookup) VLP_CUDA(cudaStreamWaitEvent(s, h->join2, 0));
    h->profiled_valid = h->profiling;
    return VLPROJ_OK;
}

int vlproj_profile_enable(vlproj_handle* h, int enable) {
    if (!h) return VLPROJ_ERR_INVALID_ARG;
    if (enable && !h->ev_begin[0]) {
        for (auto& e : h->ev_begin) VLP_CUDA(cudaEventCreate(&e));
        for (auto& e : h->ev_end) VLP_CUDA(cudaEventCreate(&e));
    }
    h->profiling = enable != 0;
    h->profiled_valid = false;
    return VLPROJ_OK;
}

int vlproj_profile_stages(vlproj_handle* h, uint32_t mask) {
    if (!h) return VLPROJ_ERR_INVALID_ARG;
    h->profile_mask = mask;
    h->profiled_valid = false;
    return VLPROJ_OK;
}

int vlproj_profile_read(vlproj_handle* h, float* ms, int n) {
    if (!h || !ms || n < 0) return VLPROJ_ERR_INVALID_ARG;
    if (!h->profiled_valid) return VLPROJ_ERR_INVALID_ARG;
    const int m = std::min(n, VLPROJ_NUM_STAGES);
    for (int i = 0; i < m; ++i) {
        float t = 0.f;
        if (h->stage_ran[i]) {
            VLP_CUDA(cudaEventSynchronize(h->ev_end[i]));
            VLP_CUDA(cudaEventElapsedTime(&t, h->ev_begin[i], h->ev_end[i]));
        }
        ms[i] = t;
    }
    return m;
}

int64_t vlproj_launch_count(vlproj_handle* h) { return h ? h->launches : VLPROJ_ERR_INVALID_ARG; }

}  // extern "C"
