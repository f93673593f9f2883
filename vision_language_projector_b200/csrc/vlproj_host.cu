// vlproj_project_host (declared in vlproj.h): features from host memory in, the batch's
// assembled rows to host memory out, with the copies pipelined against the projection.
//
// The batch is cut into runs of whole images (chunks). Chunk j uses slot j % 2 of the
// device staging (features, rows):
//   copy_in   waits until chunk j-2's projection has read the slot's features (the
//             caller's stream for the first two), copies chunk j's features in -> ev_in
//   stream    waits ev_in and until chunk j-2's rows have left the slot, projects chunk
//             j: geometry with each token's assembled row as its destination,
//             LayerNorm/convert, GEMM1, middle layers, GEMM2 straight into the slot's
//             rows, newline / separator rows                              -> ev_done
//   copy_out  waits ev_done, copies the rows to their place in rows_out      -> ev_out
// and the caller's stream finally waits for the last copies out. Host-to-device and
// device-to-host copies run on the two copy engines while the GEMMs run.
#include "host.cuh"

using namespace vlp_host;

namespace {

struct Chunk {
    int img0 = 0, n_img = 0;          // images
    int64_t view0 = 0;                // first view
    int64_t patch0 = 0;               // first patch row of the batch's features
    int64_t row0 = 0;                 // first assembled row of the batch
    size_t view_off = 0, image_off = 0;   // offsets into the uploaded descriptor tables
    Plan plan;                        // the chunk alone (patches, tokens, rows from 0)
};

int ensure_pipeline(vlproj_handle* h) {
    if (!h->copy_in) VLP_CUDA(cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking));
    if (!h->copy_out) VLP_CUDA(cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
        if (!h->ev_in[i]) VLP_CUDA(cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming));
        if (!h->ev_done[i]) VLP_CUDA(cudaEventCreateWithFlags(&h->ev_done[i], cudaEventDisableTiming));
        if (!h->ev_out[i]) VLP_CUDA(cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming));
    }
    return VLPROJ_OK;
}

// GEMM2 into the rows of a chunk, then its newline / separator rows.
int project_rows(vlproj_handle* h, const Chunk& ch, const void* features, __nv_bfloat16* rows, const void* newline,
                 const void* sep, cudaStream_t s) {
    const vlproj_config& c = h->cfg;
    const Plan& pl = ch.plan;
    int rc = run_merge_gemm1(h, pl, features, nullptr, vlp::DEST_ROW, h->H.ptr, pl.M, s,
                             h->dviews.ptr + ch.view_off);
    if (rc) return rc;
    const __nv_bfloat16* hlast = nullptr;
    rc = run_middle_layers(h, pl, s, &hlast);
    if (rc) return rc;
    CUtensorMap tmH{};
    if (encode_bf16_2d(&tmH, hlast, pl.M, c.N1, vlp::BM)) return VLPROJ_ERR_CUDA;
    GemmParams p{};
    p.M = static_cast<int>(pl.M);
    p.N = c.N2;
    p.K = c.N1;
    p.bias = h->b2;
    p.C = c.C;
    p.k = c.k;
    p.out = rows;
    p.rowdest = h->rowdest.ptr;
    p.out_rows = pl.R;
    p.fwd_status = nullptr;
    p.err = h->status;
    p.wait_ns = h->wait_ns;
    stage_begin(h, 4, s);
    ++h->launches;
    rc = launch_gemm_bn<vlp::A_TILE, vlp::EPI_SCATTER>(h, pick_bn(c.N2), h->pairs, tmH, h->tmW2, h->tmW2h, p,
                                                       s);
    if (rc) return rc;
    stage_end(h, 4, s);
    if (c.tile_tag == VLPROJ_TILE_2D && !pl.images.empty()) {
        stage_begin(h, 5, s);
        ++h->launches;
        dim3 grid(pl.max_special, static_cast<unsigned>(pl.images.size()));
        vlp::vlp_special_rows_kernel<<<grid, 128, 0, s>>>(h->dimages.ptr + ch.image_off, nullptr, pl.R,
                                                          static_cast<const __nv_bfloat16*>(newline),
                                                          static_cast<const __nv_bfloat16*>(sep), rows, pl.R, c.N2,
                                                          nullptr);
        VLP_CUDA(cudaGetLastError());
        stage_end(h, 5, s);
    }
    return VLPROJ_OK;
}

}  // namespace

extern "C" int vlproj_project_host(vlproj_handle* h, const vlproj_host_args* a, void* stream) {
    if (!h || !a || a->n_images < 0 || a->chunks < 0) return VLPROJ_ERR_INVALID_ARG;
    const vlproj_config& c = h->cfg;
    const bool tiled = c.tile_tag == VLPROJ_TILE_2D;
    const int n_images = a->n_images;
    if (n_images > 0 && (!a->features || !a->grid_hw || !a->rows_out)) return VLPROJ_ERR_INVALID_ARG;
    if (tiled && n_images > 0 &&
        (!a->newline || !a->sep || reinterpret_cast<uintptr_t>(a->newline) % 16 ||
         reinterpret_cast<uintptr_t>(a->sep) % 16))
        return VLPROJ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Plan full;
    int rc = build_plan(c, a->grid_hw, a->spatial_crop, n_images, false, h->gather_mode, &full);
    if (rc) return rc;
    if (a->rows_out_cap < full.R) return VLPROJ_ERR_INVALID_ARG;
    if (n_images == 0 || full.R == 0) return VLPROJ_OK;

    // image runs of about equal merged-token count
    std::vector<int64_t> img_view0(n_images + 1, 0), img_tok(n_images, 0), img_patch(n_images, 0);
    {
        int64_t v = 0;
        for (int i = 0; i < n_images; ++i) {
            const int nv = tiled ? 1 + a->spatial_crop[2 * i] * a->spatial_crop[2 * i + 1] : 1;
            img_view0[i] = v;
            for (int t = 0; t < nv; ++t, ++v) {
                const int hh = a->grid_hw[2 * v], ww = a->grid_hw[2 * v + 1];
                img_tok[i] += static_cast<int64_t>((hh + c.k - 1) / c.k) * ((ww + c.k - 1) / c.k);
                img_patch[i] += static_cast<int64_t>(hh) * ww;
            }
        }
        img_view0[n_images] = v;
    }
    // automatic depth: about one chunk per 16 MiB of features, 2 to 16 (measured on the
    // MoonViT, VL2, DS-ViT and 256-image batches: within 3 % of the best fixed count)
    const size_t feat_bytes = static_cast<size_t>(full.P) * c.C * (c.feat_dtype == VLPROJ_FEAT_F32 ? 4 : 2);
    const int auto_chunks = static_cast<int>(std::min<size_t>(16, std::max<size_t>(2, (feat_bytes + (8u << 20)) >> 24)));
    const int nc = std::max(1, std::min(n_images, a->chunks > 0 ? a->chunks : auto_chunks));
    const int64_t total_tok = full.M_real;
    // The first run's copy in and the last run's copy out overlap no projection, so with
    // three or more runs those two are half the size of the others.
    std::vector<double> cum(nc + 1, 0.0);
    for (int j = 0; j < nc; ++j) cum[j + 1] = cum[j] + ((nc >= 3 && (j == 0 || j == nc - 1)) ? 0.5 : 1.0);
    std::vector<Chunk> chunks;
    {
        int img = 0;
        int64_t done_tok = 0, patch = 0, row = 0;
        for (int j = 0; j < nc && img < n_images; ++j) {
            Chunk ch;
            ch.img0 = img;
            ch.view0 = img_view0[img];
            ch.patch0 = patch;
            ch.row0 = row;
            const int64_t target = static_cast<int64_t>(static_cast<double>(total_tok) * cum[j + 1] / cum[nc]);
            const int left = nc - j - 1;                       // chunks still to fill after this one
            do {
                done_tok += img_tok[img];
                patch += img_patch[img];
                ++img;
            } while (img < n_images - left && done_tok < target);
            if (j == nc - 1) {                                 // the last run takes every image left
                while (img < n_images) {
                    done_tok += img_tok[img];
                    patch += img_patch[img];
                    ++img;
                }
            }
            ch.n_img = img - ch.img0;
            rc = build_plan(c, a->grid_hw + 2 * ch.view0, a->spatial_crop ? a->spatial_crop + 2 * ch.img0 : nullptr,
                            ch.n_img, false, h->gather_mode, &ch.plan);
            if (rc) return rc;
            row += ch.plan.R;
            chunks.push_back(std::move(ch));
        }
    }

    // one upload of every chunk's view and image tables
    Plan tables;
    size_t max_patch_bytes = 0, max_rows = 0, max_m = 0;
    const size_t elem = c.feat_dtype == VLPROJ_FEAT_F32 ? 4 : 2;
    for (Chunk& ch : chunks) {
        ch.view_off = tables.views.size();
        ch.image_off = tables.images.size();
        tables.views.insert(tables.views.end(), ch.plan.views.begin(), ch.plan.views.end());
        tables.images.insert(tables.images.end(), ch.plan.images.begin(), ch.plan.images.end());
        max_patch_bytes = std::max(max_patch_bytes, static_cast<size_t>(ch.plan.P) * c.C * elem);
        max_rows = std::max(max_rows, static_cast<size_t>(ch.plan.R));
        max_m = std::max(max_m, static_cast<size_t>(ch.plan.M));
    }
    rc = ensure_pipeline(h);
    if (rc) return rc;
    for (int i = 0; i < 2; ++i)
        if (h->stage_feat[i].ensure(max_patch_bytes) || h->stage_rows[i].ensure(max_rows * c.N2))
            return VLPROJ_ERR_CUDA;
    if (h->H.ensure(max_m * c.N1) || (c.depth > 2 && h->H2.ensure(max_m * c.N1))) return VLPROJ_ERR_CUDA;
    rc = upload_plan(h, tables, s);
    if (rc) return rc;
    h->profiled_valid = false;
    for (bool& r : h->stage_ran) r = false;

    // the copy streams start after everything already on the caller's stream
    VLP_CUDA(cudaEventRecord(h->fork, s));
    VLP_CUDA(cudaStreamWaitEvent(h->copy_in, h->fork, 0));
    const uint8_t* feat_host = static_cast<const uint8_t*>(a->features);
    uint8_t* rows_host = static_cast<uint8_t*>(a->rows_out);
    const size_t row_bytes = static_cast<size_t>(c.N2) * 2;
    for (size_t j = 0; j < chunks.size(); ++j) {
        const Chunk& ch = chunks[j];
        const int slot = static_cast<int>(j & 1);
        if (j >= 2) VLP_CUDA(cudaStreamWaitEvent(h->copy_in, h->ev_done[slot], 0));
        VLP_CUDA(cudaMemcpyAsync(h->stage_feat[slot].ptr, feat_host + ch.patch0 * c.C * elem,
                                 static_cast<size_t>(ch.plan.P) * c.C * elem, cudaMemcpyHostToDevice, h->copy_in));
        VLP_CUDA(cudaEventRecord(h->ev_in[slot], h->copy_in));
        VLP_CUDA(cudaStreamWaitEvent(s, h->ev_in[slot], 0));
        if (j >= 2) VLP_CUDA(cudaStreamWaitEvent(s, h->ev_out[slot], 0));
        rc = project_rows(h, ch, h->stage_feat[slot].ptr, h->stage_rows[slot].ptr, a->newline, a->sep, s);
        if (rc) return rc;
        VLP_CUDA(cudaEventRecord(h->ev_done[slot], s));
        VLP_CUDA(cudaStreamWaitEvent(h->copy_out, h->ev_done[slot], 0));
        VLP_CUDA(cudaMemcpyAsync(rows_host + ch.row0 * row_bytes, h->stage_rows[slot].ptr,
                                 static_cast<size_t>(ch.plan.R) * row_bytes, cudaMemcpyDeviceToHost, h->copy_out));
        VLP_CUDA(cudaEventRecord(h->ev_out[slot], h->copy_out));
    }
    for (size_t j = 0; j < std::min<size_t>(2, chunks.size()); ++j)
        VLP_CUDA(cudaStreamWaitEvent(s, h->ev_out[(chunks.size() - 1 - j) & 1], 0));
    h->profiled_valid = h->profiling;
    return VLPROJ_OK;
}
