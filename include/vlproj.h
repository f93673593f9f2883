/*
 * vlproj - vision-to-language projector for NVIDIA B200 (sm_100a).
 *
 * The bridge between a vision tower and a language model's embedding
 * sequence, as described on the pages studied for this library:
 *
 *   1. space-to-depth: each k x k neighbourhood of a view's patch grid becomes
 *      one token of k*k*C features, grid zero-padded at the high end to a
 *      multiple of k, features ordered channel-outermost c*k*k + dy*k + dx
 *      ("port DeepSeek-VL2", Projector (downsample_mlp_gelu) steps 1-2;
 *      "La voie visuelle", section "Le pixel-unshuffle 3x3");
 *   2. optional pre-merge LayerNorm over each patch's C features (the MoonViT
 *      PatchMerger: "DeepSeek-V4-Flash-Vision-BF16", first section);
 *   3. Linear -> GELU -> Linear, weights stored (out, in)
 *      ("port DeepSeek-VL2", Projector step 3 and Safetensors weight keys);
 *   4. for tile tag "2D": global view rows each closed by a learned newline,
 *      one view separator, then the local tiles laid side by side, rows closed
 *      by a newline ("port DeepSeek-VL2", Tile-sequence assembly);
 *   5. the assembled rows overwrite the embedding rows that hold the image
 *      placeholder id, in order ("port DeepSeek-VL2", end of Tile-sequence
 *      assembly; image_token_index 100015);
 *   6. the gradients of the projector's parameters and of the features, for
 *      training the projector between a frozen tower and a frozen language model
 *      ("DeepSeek-V4-Flash-Vision-BF16", opening section): vlproj_backward.
 *
 * Number formats: bf16 operands, fp32 accumulation, bf16 hidden activation
 * and bf16 output rows. Everything below runs on the GPU; there is no CPU path.
 *
 * Conventions
 *   - Every call returns a vlproj status code (>= 0 success, < 0 error) unless
 *     stated otherwise. Errors found on the host return before any launch and
 *     leave every buffer untouched.
 *   - Device pointers are raw CUDA device addresses; host pointers are plain
 *     CPU memory. The library never takes ownership of a caller's buffer.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Work is enqueued asynchronously; the caller keeps every
 *     borrowed device buffer alive until that stream's work completes.
 *   - A handle is bound to the device that was current at vlproj_create and
 *     is not thread-safe: one thread at a time per handle. Its calls share the
 *     handle's scratch buffers, so successive calls go on one stream (or on
 *     streams the caller orders); calls on different handles are independent.
 */
#ifndef VLPROJ_H
#define VLPROJ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define VLPROJ_OK                 0
#define VLPROJ_ERR_INVALID_ARG   (-1) /* bad pointer, size, shape or layout */
#define VLPROJ_ERR_UNSUPPORTED   (-2) /* projector variant the library does not build (the
                                         pages ask for a loud error on these: tile tag "1D",
                                         token pooling, another projector type) */
#define VLPROJ_ERR_CUDA          (-3) /* a CUDA runtime/driver call failed */
#define VLPROJ_ERR_TOKEN_COUNT   (-4) /* device found: placeholder count != assembled rows;
                                         nothing was written to out_embeds */
#define VLPROJ_ERR_TIMEOUT       (-5) /* device found: a bounded wait inside a kernel ran out */

/* ---- configuration ----------------------------------------------------- */
enum { VLPROJ_FEAT_BF16 = 0, VLPROJ_FEAT_F32 = 1 };
enum { VLPROJ_TILE_NONE = 0, VLPROJ_TILE_2D = 1, VLPROJ_TILE_1D = 2 /* rejected */ };
enum { VLPROJ_GLOBAL_HEAD = 0, VLPROJ_GLOBAL_TAIL = 1 };
enum { VLPROJ_ORDER_CHANNEL_OUTER = 0,   /* W1 input index c*k*k + dy*k + dx (the pages' order) */
       VLPROJ_ORDER_POSITION_OUTER = 1 }; /* W1 input index (dy*k + dx)*C + c */

typedef struct vlproj_config {
    int32_t k;              /* merge factor: 1, 2 or 3 */
    int32_t C;              /* vision feature width; multiple of 64 */
    int32_t N1;             /* MLP hidden width; multiple of 64 */
    int32_t N2;             /* output embedding width (n_embed); multiple of 32 */
    int32_t depth;          /* number of Linear layers, 2..8: depth > 2 inserts depth-2 pairs
                               GELU -> Linear(N1 -> N1) between the first and the last
                               ("port DeepSeek-VL2", Projector step 3) */
    int32_t has_ln;         /* 1: pre-merge LayerNorm over C, biased variance */
    float   ln_eps;         /* LayerNorm epsilon (1e-5 when <= 0) */
    int32_t feat_dtype;     /* VLPROJ_FEAT_BF16 or VLPROJ_FEAT_F32 features */
    int32_t k_order;        /* column order of W1 as passed (see enum) */
    int32_t tile_tag;       /* VLPROJ_TILE_NONE or VLPROJ_TILE_2D */
    int32_t global_view_pos;/* VLPROJ_GLOBAL_HEAD or VLPROJ_GLOBAL_TAIL (2D tiling) */
    int32_t token_pooling;  /* must be 0 */
    /* Parameters, all DEVICE pointers, read once by vlproj_create (which copies
     * them into storage the handle owns and synchronises, so the caller may free
     * its buffers when create returns). */
    const void*  W1;        /* bf16 [N1][k*k*C], stored (out, in) */
    const float* b1;        /* fp32 [N1], or NULL for zeros */
    const void*  W2;        /* bf16 [N2][N1], stored (out, in) */
    const float* b2;        /* fp32 [N2], or NULL for zeros */
    const float* ln_gamma;  /* fp32 [C] when has_ln, else ignored */
    const float* ln_beta;   /* fp32 [C] when has_ln, else ignored */
    /* depth > 2 only: HOST arrays of depth-2 DEVICE pointers, layer order */
    const void* const*  W_mid;   /* each bf16 [N1][N1], stored (out, in) */
    const float* const* b_mid;   /* each fp32 [N1]; the array or an entry may be NULL (zeros) */
} vlproj_config;

typedef struct vlproj_handle vlproj_handle;

/* Create a projector on the current device. Validates cfg (VLPROJ_ERR_UNSUPPORTED
 * for depth outside 2..8, tile tag "1D", token pooling, k outside 1..3; INVALID_ARG for
 * widths that break the alignment rules above or NULL weights), allocates the
 * owned weight copies and permutes W1's columns into the kernel's gather order
 * (an exact permutation of bf16 values). On success *out holds the handle. */
int vlproj_create(const vlproj_config* cfg, vlproj_handle** out);

/* Run the whole bridge for one batch, asynchronously on `stream`.
 *   features     DEVICE, packed channel-last patch features of every view, views
 *                back to back: view v holds grid_hw[v][0]*grid_hw[v][1] rows of C
 *                values (bf16 or fp32 per cfg), rows row-major over (h, w).
 *                For 2D tiling the views of an image are [global, local tiles
 *                row-major]; all views of one image share one grid.
 *   grid_hw      HOST, int32 [n_views][2] = (h, w) per view; n_views = n_images
 *                untiled, sum(1 + tw*th) when tiled.
 *   spatial_crop HOST, int32 [n_images][2] = (tw, th) per image (width count
 *                first), or NULL when cfg.tile_tag == VLPROJ_TILE_NONE.
 *   n_images     number of images (0 = text only: the call only checks that no
 *                placeholder is present).
 *   input_ids    DEVICE, int64 [n_ids], all sequences flattened (B*S).
 *   image_token_id  the placeholder id (100015 in the DeepSeek-VL family).
 *   newline, sep DEVICE, bf16 [N2] each when tiled, else ignored (may be NULL).
 *   out_embeds   DEVICE, bf16 [n_ids][N2], in/out: only placeholder rows are
 *                written; every other row is left as it was.
 * Image i's rows go to the placeholders in order: the j-th placeholder over the
 * flattened ids receives assembled row j. The placeholder count is checked on the
 * device against the closed-form row count; on mismatch nothing is written and
 * VLPROJ_ERR_TOKEN_COUNT is latched (see vlproj_status). */
int vlproj_forward(vlproj_handle* h,
                   const void* features,
                   const int32_t* grid_hw,
                   const int32_t* spatial_crop,
                   int32_t n_images,
                   const int64_t* input_ids, int64_t n_ids,
                   int64_t image_token_id,
                   const void* newline, const void* sep,
                   void* out_embeds,
                   void* stream);

/* Extended forward: everything vlproj_forward does, plus two optional outputs.
 *   embed_table  DEVICE bf16 [vocab][N2], or NULL. When given, every row i of out_embeds
 *                whose id is not the placeholder is written as embed_table[input_ids[i]]:
 *                the language model's token-embedding lookup that the assembled rows then
 *                overwrite at the placeholders ("port DeepSeek-VL2", end of Tile-sequence
 *                assembly), done in the same call on a side stream while the GEMMs run.
 *                An id outside [0, vocab) gives a zero row and latches
 *                VLPROJ_ERR_INVALID_ARG (read with vlproj_status).
 *   rows_out     DEVICE bf16 [rows_out_cap][N2], or NULL. When given, the R assembled rows
 *                of the batch (projected rows, newlines and separators, in placeholder
 *                order) are also written here contiguously; rows_out_cap must be >= R
 *                (vlproj_image_rows gives R), else VLPROJ_ERR_INVALID_ARG before any
 *                launch. Nothing is written when the placeholder count check fails.
 * All other fields mean what the arguments of vlproj_forward mean. */
typedef struct vlproj_forward_args {
    const void*    features;
    const int32_t* grid_hw;
    const int32_t* spatial_crop;
    int32_t        n_images;
    const int64_t* input_ids;
    int64_t        n_ids;
    int64_t        image_token_id;
    const void*    newline;
    const void*    sep;
    void*          out_embeds;
    const void*    embed_table;
    int64_t        vocab;
    void*          rows_out;
    int64_t        rows_out_cap;
} vlproj_forward_args;
int vlproj_forward_ex(vlproj_handle* h, const vlproj_forward_args* args, void* stream);

/* ---- host memory in, host memory out -----------------------------------
 * The projected rows of a batch whose features are in host memory, written to host
 * memory: the same rows as vlproj_forward_ex's rows_out (every image's assembled rows,
 * newlines and separators included, images in order; "port DeepSeek-VL2",
 * Tile-sequence assembly), without the embedding buffer. The batch is cut into
 * `chunks` runs of whole images of about equal token count, the first and the last
 * about half the others when there are three or more, since their copies overlap no
 * projection (0 = automatic); chunk j's
 * features are copied to the device while chunk j-1 is projected and chunk j-2's rows
 * are copied back, on copy streams of the handle, so PCIe traffic in both directions
 * overlaps the GEMMs. Work is enqueued behind `stream`; the call returns without
 * waiting, and `stream` completes only after the last rows have reached rows_out.
 *   features   HOST, as for vlproj_forward (packed views, feat_dtype); page-locked
 *              memory (cudaHostAlloc / cudaHostRegister) for the copies to overlap.
 *   grid_hw, spatial_crop, n_images, newline, sep: as for vlproj_forward.
 *   rows_out   HOST bf16 [rows_out_cap][N2], rows_out_cap >= R (vlproj_image_rows),
 *              page-locked for the copies to overlap.
 *   chunks     pipeline depth in image runs; 0 picks about one run per 16 MiB of
 *              features, 2 to 16; never more runs than images.
 * Both host buffers must stay valid and untouched until `stream` has completed.
 * Errors: VLPROJ_ERR_INVALID_ARG for inconsistent shapes, a small rows_out_cap or a
 * NULL buffer, before any work is enqueued. */
typedef struct vlproj_host_args {
    const void*    features;
    const int32_t* grid_hw;
    const int32_t* spatial_crop;
    int32_t        n_images;
    const void*    newline;
    const void*    sep;
    void*          rows_out;
    int64_t        rows_out_cap;
    int32_t        chunks;
} vlproj_host_args;
int vlproj_project_host(vlproj_handle* h, const vlproj_host_args* args, void* stream);

/* ---- backward -----------------------------------------------------------
 * Gradients of the projector for one batch. The bridge is trained with the vision
 * tower and the language model frozen, so the projector's parameters are the only
 * trained ones ("DeepSeek-V4-Flash-Vision-BF16", opening section: a 40,119,040-
 * parameter projector trained between the frozen tower and backbone, with forward /
 * backward gates passed in BF16). Given d_out, the gradient of the loss with respect
 * to the combined embedding buffer that vlproj_forward writes, this returns the
 * gradients of W1, b1, W2, b2, the LayerNorm gamma / beta, the newline and separator
 * rows, and of the features, by the chain rule through the forward steps:
 *   dY[m]  = d_out[placeholder row of merged token m]
 *   dW2    = dY^T H,  db2 = sum_m dY[m]
 *   dP     = (dY W2) * GELU'(P),  P = A W1^T + b1 (recomputed from the features)
 *   dW1    = dP^T A,  db1 = sum_m dP[m]
 *   dA     = dP W1, folded back through the space-to-depth onto the patches, then
 *            through the LayerNorm: dgamma, dbeta and d_features
 *   dnewline / dsep = sums of d_out over the newline / separator rows.
 * With depth > 2 ("port DeepSeek-VL2", Projector step 3) the chain runs through the
 * middle GELU + Linear(N1 -> N1) layers the same way: dW_mid[i] = dP_(i+2)^T H_(i+1),
 * db_mid[i] = sum_m dP_(i+2)[m], dP_(i+1) = (dP_(i+2) W_mid[i]) * GELU'(P_(i+1)), where
 * layer 1 is the first Linear and layer `depth` the last.
 * The bf16 rounding points of the forward (A and every hidden activation) pass
 * gradients unchanged; A and the hidden activations are the forward's bf16 values,
 * each dP is rounded to bf16 once, and with a LayerNorm so is dA (fp32 accumulation
 * throughout).
 *
 *   features, grid_hw, spatial_crop, n_images, input_ids, n_ids, image_token_id:
 *                 as for vlproj_forward (the same batch the loss was computed on).
 *   d_out         DEVICE bf16 [n_ids][N2], 16-byte aligned. Rows of text tokens are
 *                 ignored.
 *   d_W1 .. d_features  DEVICE fp32 outputs, overwritten (not accumulated), each
 *                 16-byte aligned, or NULL when not wanted (work that only feeds
 *                 unwanted outputs is skipped):
 *                   d_W1 [N1][k*k*C] (columns in the config's k_order), d_b1 [N1],
 *                   d_W2 [N2][N1], d_b2 [N2], d_gamma [C], d_beta [C] (LayerNorm only),
 *                   d_newline [N2], d_sep [N2] (2D tiling only), d_features [P][C].
 *   d_W_mid, d_b_mid  depth > 2: HOST arrays of depth - 2 DEVICE fp32 pointers
 *                 (d_W_mid[i] [N1][N1], d_b_mid[i] [N1]), or NULL; an entry may be NULL.
 *                 Ignored for depth 2.
 * Scratch: about 2 * M * (2*N1*(depth - 1) + N1*(depth - 2) + 2*N1 + 2*N2 + 3*k*k*C)
 * bytes (M merged tokens), kept in the handle. Errors as for vlproj_forward; when the
 * placeholder count check fails every gradient is written as zero and
 * VLPROJ_ERR_TOKEN_COUNT is latched. */
typedef struct vlproj_backward_args {
    const void*    features;
    const int32_t* grid_hw;
    const int32_t* spatial_crop;
    int32_t        n_images;
    const int64_t* input_ids;
    int64_t        n_ids;
    int64_t        image_token_id;
    const void*    d_out;
    float*         d_W1;
    float*         d_b1;
    float*         d_W2;
    float*         d_b2;
    float*         d_gamma;
    float*         d_beta;
    float*         d_newline;
    float*         d_sep;
    float*         d_features;
    float* const*  d_W_mid;
    float* const*  d_b_mid;
} vlproj_backward_args;
int vlproj_backward(vlproj_handle* h, const vlproj_backward_args* args, void* stream);

/* Stage output for inspection: the bf16 hidden activation H = GELU(A W1^T + b1)
 * of every merged token, views in order, tokens row-major inside a view.
 * hidden is DEVICE bf16 [M][N1], M = sum over views of ceil(h/k)*ceil(w/k). */
int vlproj_hidden(vlproj_handle* h, const void* features, const int32_t* grid_hw,
                  int32_t n_views, void* hidden, void* stream);

/* Synchronise `stream`, then return the first device-found error latched since the
 * last call (VLPROJ_OK if none) and clear it. */
int vlproj_status(vlproj_handle* h, void* stream);

/* Free the handle and everything it owns (synchronises its device first). NULL is a no-op. */
void vlproj_destroy(vlproj_handle* h);

/* Host only, no device work: closed-form placeholder count of each image
 * (untiled: ceil(h/k)*ceil(w/k); 2D: h'(w'+1) + 1 + (th h')(tw w'+1), from
 * "port DeepSeek-VL2", Processor step 7). Writes rows_out[n_images] when not
 * NULL and returns the total (>= 0) or an error code (< 0). */
int64_t vlproj_image_rows(const vlproj_config* cfg, const int32_t* grid_hw,
                          const int32_t* spatial_crop, int32_t n_images, int64_t* rows_out);

/* How GEMM1 fetches each merged token's k x k neighbourhood from the features:
 *   VLPROJ_GATHER_AUTO    (default) with a pre-merge LayerNorm or fp32 features, the
 *                         LayerNorm / convert pass writes its bf16 output directly in
 *                         merged-token order and GEMM1 reads it as a plain matrix;
 *                         otherwise BOX when every view has the same grid, k divides it
 *                         and w' = w/k divides 128; else IM2COL when every view has the
 *                         same grid; else CPASYNC (measured faster for mixed grids).
 *                         BOX, IM2COL and CPASYNC apply a LayerNorm pass in patch order
 *                         and gather from its output;
 *   VLPROJ_GATHER_FUSED   four producer warps per CTA of GEMM1 write the merged (and
 *                         LayerNorm'd or converted) operand rows into device memory, in
 *                         256-row blocks by tap, a little ahead of the TMA tile loads that
 *                         read them back (each waits for its block's tap to be complete):
 *                         one kernel, the copy's writes overlapped with the MMAs;
 *   VLPROJ_GATHER_MERGED  a LayerNorm / convert / merge pass writes the merged operand
 *                         first, then GEMM1 reads it by TMA tiles;
 *   VLPROJ_GATHER_THREADS four extra warps per CTA gather each row by 16-byte cp.async
 *                         (zero-filled pad), on CTA pairs too; with a LayerNorm on bf16
 *                         features they normalise each landed stage in shared memory
 *                         from per-patch statistics (8 bytes per patch), so no
 *                         normalised or merged copy of the features exists in memory;
 *   VLPROJ_GATHER_BOX     one 5D tiled TMA box per K-block: the features seen as
 *                         (c, dx, j, dy, merged row); falls back to IM2COL when the
 *                         grids are not regular as above;
 *   VLPROJ_GATHER_IM2COL  TMA im2col loads, the merge seen as a k x k, stride-k
 *                         convolution window walk with hardware zero fill of the
 *                         high-end pad; one map for a batch of same-shape views, else
 *                         one map per view with each view's rows padded to 32;
 *   VLPROJ_GATHER_CPASYNC 16-byte cp.async copies per row (zero-filled pad).
 * All give the same bits. */
enum {
    VLPROJ_GATHER_IM2COL = 0,
    VLPROJ_GATHER_CPASYNC = 1,
    VLPROJ_GATHER_AUTO = 2,
    VLPROJ_GATHER_BOX = 3,
    VLPROJ_GATHER_THREADS = 4,
    VLPROJ_GATHER_FUSED = 5,
    VLPROJ_GATHER_MERGED = 6
};
int vlproj_set_gather_mode(vlproj_handle* h, int mode);

/* GEMM tile shape. enable = 1 (default): 256 x 256 tiles run on pairs of CTAs
 * (cta_group::2 MMA; each CTA stages its 128 rows of A and half of B, so B crosses
 * L2 once per pair) wherever N >= 256 and A arrives by TMA; enable = 0: 128 x 256
 * tiles on single CTAs. Both give the same bits. */
int vlproj_set_tile_pairs(vlproj_handle* h, int enable);

/* Raster of the GEMMs' persistent tile loop (forward and backward): output tiles are
 * walked in bands of N-blocks whose slice of the operand B fits in `bytes`; inside a band
 * the M-block advances slowest, so the CTAs running together share their A tiles and the
 * band's B stays in L2. A larger budget means fewer bands, so A is read from memory fewer
 * times. 0 = the default: 64 MB (about half of the 126 MB L2), and where a single
 * N-block's slice is larger than that (the weight gradients of big batches, K = tokens)
 * bands of about sqrt(number of CTAs running at once) N-blocks, so a wave reads the
 * fewest operand panels. The result does not depend on it (each output's K order is
 * fixed). bytes < 0 is rejected. */
int vlproj_set_raster_budget(vlproj_handle* h, int64_t bytes);

/* Order in which the GEMMs' persistent CTAs (or CTA pairs) take their output tiles.
 * VLPROJ_TILE_ORDER_DYNAMIC: each takes the next tile of the raster order from a counter
 * in device memory when it starts one, so tiles start in raster order however the CTAs'
 * speeds differ, and the tiles that share an A block or a B panel run at the same time
 * and read it from L2. VLPROJ_TILE_ORDER_STATIC: CTA u runs tiles u, u + CTAs, u + 2 CTAs,
 * ... (over hundreds of waves the CTAs drift apart and re-read operands from DRAM).
 * VLPROJ_TILE_ORDER_AUTO (the default): dynamic for GEMMs whose A operand is gathered
 * (the merge-gather feeds) and for those with at least 64 waves' work of 64-K-block
 * tiles, static for the other plain-matrix GEMMs (measured faster so). The handle holds 64 counters, zeroed by
 * vlproj_create and left zeroed by every GEMM; calls on one handle must not run
 * concurrently (as for its other scratch). Every order gives the same bits (each
 * output's K order is fixed). Other values are rejected with VLPROJ_ERR_INVALID_ARG. */
enum { VLPROJ_TILE_ORDER_STATIC = 0, VLPROJ_TILE_ORDER_AUTO = 1, VLPROJ_TILE_ORDER_DYNAMIC = 2 };
int vlproj_set_tile_order(vlproj_handle* h, int order);

/* Host only, no device work: the processor's tiling choices for the 2D tile scheme
 * ("port DeepSeek-VL2", Processor steps 1, 2, 6, 7). For each image of one request,
 * with original size image_wh[i] = (w0, h0) in pixels (width first):
 *   - cropping applies only when the request has at most 2 images (else grid 1x1);
 *   - with cropping, the candidate (W, H) in candidates[n_candidates][2] maximising
 *     effective = min(floor(w0*s)*floor(h0*s), w0*h0), s = min(W/w0, H/h0) (IEEE
 *     double), ties to the least wasted area W*H - effective, first candidate on a
 *     full tie;
 *   - spatial_crop_out[i] = (tw, th) = (W / image_size, H / image_size);
 *   - rows_out[i] = h'(w'+1) + 1 + (th h')(tw w'+1) placeholders, h' = w' =
 *     ceil(floor(image_size / patch_size) / downsample).
 * Returns the number of views, sum of (1 + tw*th), or an error code (< 0). Each view
 * is one image_size x image_size tile with a floor(image_size/patch_size) square grid. */
int64_t vlproj_plan_tiles(const int32_t* image_wh, int32_t n_images, const int32_t* candidates, int32_t n_candidates,
                          int32_t image_size, int32_t patch_size, int32_t downsample, int32_t* spatial_crop_out,
                          int64_t* rows_out);

/* Bound (nanoseconds) on every wait inside this handle's kernels; 0 restores the
 * default (2 s). A wait that runs out ends its kernel early with
 * VLPROJ_ERR_TIMEOUT latched; tests use a tiny bound to exercise that path. */
int vlproj_set_wait_limit(vlproj_handle* h, uint64_t ns);

/* ---- tracing ------------------------------------------------------------
 * Stage timing with CUDA events recorded on the launching stream around each
 * kernel of vlproj_forward / vlproj_backward. Stages, in order:
 *   forward   0 placeholder index (and GEMM2's row map), 1 geometry (gather data; not
 *             launched when GEMM1 reads none and no row table is wanted, e.g. with the
 *             merged LayerNorm or the 5D box gather), 2 LayerNorm/convert, 3 GEMM1
 *             (merge + MLP first layer + GELU), 4 GEMM2 (second layer + scatter),
 *             5 newline/separator rows;
 *   backward  6 placeholder index + geometry, 7 LayerNorm-merge (A), 8 GEMM1
 *             recompute (GELU' and H^T), 9 dY gather, 10 dH GEMM (dP), 11 dW2 GEMM,
 *             12 dW1 GEMM + its column reorder, 13 dA GEMM, 14 bias sums + LayerNorm backward +
 *             newline/separator gradients.
 * Off by default; enabling adds two event records per stage that runs. */
#define VLPROJ_NUM_STAGES 15
int vlproj_profile_enable(vlproj_handle* h, int enable);

/* Which stages record events while profiling is on: bit i = stage i (default: all).
 * Each timed stage adds two event records to the stream, which separate its kernel
 * from its neighbours; timing only the stages of interest keeps that cost off the
 * others. Stages outside the mask read 0 in vlproj_profile_read. */
int vlproj_profile_stages(vlproj_handle* h, uint32_t mask);

/* Synchronise the stream of the most recent profiled call and write the elapsed
 * milliseconds of each stage into ms[0 .. min(n, VLPROJ_NUM_STAGES)); a stage that did
 * not run reads 0. Returns the number of values written, or an error code. */
int vlproj_profile_read(vlproj_handle* h, float* ms, int n);

/* Number of kernels this handle has launched since it was created (all entry points). */
int64_t vlproj_launch_count(vlproj_handle* h);

/* ---- placeholder index without allocation ------------------------------
 * The pages have no counterpart to this entry point; it serves callers of this
 * library that must not allocate device memory when they call it: code where an
 * allocation would synchronise the device or break a latency budget, or code with
 * no allocator of its own to hand (a plain C caller that only borrows buffers).
 *
 * Writes positions[j] = flat index of the j-th element of input_ids equal to
 * image_token_id (in order, for j < max_positions) and *count = how many there are,
 * asynchronously on `stream`: the same step as the placeholder index of
 * vlproj_forward, needing no handle. input_ids: DEVICE int64 [n_ids]; positions:
 * DEVICE int32 [max_positions]; count: DEVICE int64 [1].
 * It calls no allocator: its only scratch (one int32 per 4096 ids, then their total)
 * is a fixed array in the library's device memory, VLPROJ_NOALLOC_MAX_IDS / 4096 + 1
 * entries (about 64 KB), held by every GPU that loads the library until the process
 * exits. The work is linear in n_ids (count, one prefix-sum pass, compact). n_ids beyond
 * VLPROJ_NOALLOC_MAX_IDS returns VLPROJ_ERR_INVALID_ARG before any launch.
 * The first call on each device looks up that device's copy of the array (with the
 * device current) and should come before any stream capture. All calls share the
 * array: calls that overlap on the same GPU race on it. */
#define VLPROJ_NOALLOC_MAX_IDS (64 * 1024 * 1024)
int vlproj_placeholder_index_noalloc(const int64_t* input_ids, int64_t n_ids, int64_t image_token_id,
                                     int32_t* positions, int64_t max_positions, int64_t* count, void* stream);

/* Human-readable name of a status code (static string). */
const char* vlproj_strerror(int code);

/* Library version string, e.g. "vlproj 0.1 sm_100a". */
const char* vlproj_version(void);

#ifdef __cplusplus
}
#endif
#endif /* VLPROJ_H */
