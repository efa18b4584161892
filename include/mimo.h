/*
 * mimo.h -- C ABI of the B200 MiMo-V2 image preprocessing library.
 *
 * The library turns decoded 8-bit images into the patch rows the MiMo-V2
 * vision tower consumes, on the GPU, in one fused kernel per batch. The
 * operation is the pixel path of MimoV2ImageProcessor (NeMo Automodel page
 * "nemo_automodel.components.models.mimo_v2_flash.processing", class
 * MimoV2ImageProcessor and its __call__; restated on docs.rs
 * "cortiq_engine::mimo_vision", conventions list and prepare_image):
 *
 *   smart_resize geometry (factor = patch_size * merge_size = 32)
 *   -> RGBA composited onto white (function _to_rgb), alpha dropped
 *   -> uint8 to float on the 0..255 scale
 *   -> bilinear resize, align_corners=False, no antialias, no 8-bit rounding
 *   -> (x - 255*mean_c) / (255*std_c)
 *   -> the frame duplicated to temporal_patch_size = 2 frames
 *   -> rows of 3*2*16*16 = 1536 values laid out (c, tt, py, px),
 *      rows ordered (t, block row, block col, mh, mw) (merge-block order)
 *   -> optionally the column-order row permutation (column_permutation:
 *      merge units listed by (t, block col, block row), perm[dst] = src).
 *
 * Conventions for every entry point:
 *   - Return value: a mimo_status (0 = MIMO_OK). Every argument problem the
 *     host can see is reported before anything is launched or copied. The
 *     device code contains no traps. The pixel kernels wait only for their
 *     own CTA's or warp's copies and barriers, never on other CTAs. The
 *     patch-embedding kernel's waits are bounded and report through d_error.
 *   - Ownership: the caller owns every buffer. The library never allocates
 *     or frees device memory at run time. Between calls it keeps:
 *       - the fixed staging area of mimo_preprocess_batch_host_noalloc;
 *       - the two streams and events of mimo_preprocess_embed, per host
 *         thread and device;
 *       - cached device attributes (SM count, occupancy, shared-memory
 *         opt-in).
 *   - "d_" pointers are device pointers, "h_" pointers host pointers; the
 *     other arrays (sizes, offsets) are host arrays read during the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Device work is asynchronous on it unless stated otherwise.
 *   - Only the geometry knobs patch_size = 16, temporal_patch_size = 2 and
 *     merge_size = 2 are implemented on the GPU (the processor's defaults);
 *     other values return MIMO_EUNSUPPORTED.
 */
#ifndef MIMO_H_
#define MIMO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MIMO_OK = 0,
    MIMO_EINVAL = 1,        /* null pointer, negative count, non-positive size, bad knob */
    MIMO_EASPECT = 2,       /* long/short side above 200 with the short side >= factor   */
    MIMO_EDEGENERATE = 3,   /* the max_pixels shrink rounds a side down to zero          */
    MIMO_ECHANNELS = 4,     /* channels other than 3 (RGB) or 4 (RGBA)                  */
    MIMO_EUNSUPPORTED = 5,  /* patch/temporal/merge other than 16/2/2, or std <= 0       */
    MIMO_EALIGN = 6,        /* a source offset or output pointer is not 16-byte aligned  */
    MIMO_ECAPACITY = 7,     /* an output or staging buffer is too small for the batch    */
    MIMO_EOVERFLOW = 8,     /* a size does not fit the index types (see each call)       */
    MIMO_ECUDA = 9,         /* a CUDA runtime call failed (launch or copy)               */
    MIMO_ERANGE = 10,       /* an image reaches past the end of the source buffer        */
    MIMO_ELIMIT = 11        /* an image does not fit the fixed no-allocation staging area */
} mimo_status;

typedef enum {
    MIMO_F32 = 0,   /* float32 patch values (the processor's own output type)   */
    MIMO_BF16 = 1   /* bfloat16, rounded to nearest-even from the float32 value */
} mimo_dtype;

typedef enum {
    MIMO_ORDER_MERGE = 0,  /* rows by (t, block row, block col, mh, mw): the processor's order */
    MIMO_ORDER_COLUMN = 1  /* merge units by (t, block col, block row), a unit's 4 rows kept
                              together (cortiq page, conventions: column-order windows);
                              the same rows as MIMO_ORDER_MERGE gathered with the column
                              permutation */
} mimo_row_order;

/*
 * Processor knobs (class MimoV2ImageProcessor constructor; per-call
 * min_pixels / max_pixels overrides of __call__ are expressed by passing a
 * struct with other bounds). Statistics are always caller-supplied: the page
 * reads them from the checkpoint (ImageNet for MiMo-V2.6, CLIP for V2.5).
 */
typedef struct {
    int32_t patch_size;           /* 16 */
    int32_t temporal_patch_size;  /* 2  */
    int32_t merge_size;           /* 2  */
    int32_t reserved;             /* must be 0 */
    int64_t min_pixels;           /* 8192    (lower bound on resized area) */
    int64_t max_pixels;           /* 8388608 (upper bound on resized area) */
    float image_mean[3];          /* per-channel mean on the 0..1 scale    */
    float image_std[3];           /* per-channel std on the 0..1 scale, > 0 */
} mimo_params;

/* Fills the constructor defaults: 16/2/2, 8192, 8388608, ImageNet
 * mean (0.485, 0.456, 0.406) and std (0.229, 0.224, 0.225). */
void mimo_params_default(mimo_params *p);

/*
 * smart_resize (processing page, function smart_resize; cortiq page,
 * smart_resize). Resized (height, width), both multiples of `factor`:
 *  - a side below `factor` first scales both sides so the short side equals
 *    `factor` and the long side becomes floor(long * factor / short), the
 *    integer sizes the MiMo processor (sglang semantics) continues with; that
 *    branch skips the aspect guard;
 *  - otherwise long/short > 200 -> MIMO_EASPECT;
 *  - each side rounds to the nearest multiple of factor (exact halves to
 *    even); an area above max_pixels shrinks by sqrt(area/max_pixels) with
 *    floor (a zero side -> MIMO_EDEGENERATE), an area below min_pixels grows
 *    by sqrt(min_pixels/area) with ceil.
 * Host only. Errors: MIMO_EINVAL for non-positive sizes/factor, null outputs.
 */
int mimo_smart_resize(int64_t height, int64_t width, int64_t factor,
                      int64_t min_pixels, int64_t max_pixels,
                      int64_t *out_height, int64_t *out_width);

/*
 * get_number_of_image_patches (processing page): grid_h * grid_w of the
 * resized image, counted before each merge_size**2 patches merge into one
 * token (vision tokens = *out_patches / 4). Host only.
 */
int mimo_num_patches(int64_t height, int64_t width, const mimo_params *p, int64_t *out_patches);

/*
 * Batch plan (the __call__ batch assembly: per-image rows concatenated,
 * image_grid_thw of shape [n, 3]). Host only.
 *   heights/widths: [n] source sizes.
 *   grid_thw:       out, [n*3] int64, rows (1, H'/16, W'/16).
 *   row_offsets:    out, [n+1] int64, first output row of each image; the
 *                   last entry is the total number of rows.
 * The first image whose geometry fails decides the returned status. A
 * resized side of 2^30 pixels or more is MIMO_EOVERFLOW (reachable only with
 * a max_pixels far above the default).
 */
int mimo_plan_batch(int32_t n, const int32_t *heights, const int32_t *widths,
                    const mimo_params *p, int64_t *grid_thw, int64_t *row_offsets);

/*
 * The fused pixel path for a batch, on the GPU.
 *   d_src:        device, packed interleaved HWC uint8 images, 16-byte aligned.
 *   src_bytes:    size of the d_src buffer; every image must lie inside it
 *                 (MIMO_ERANGE otherwise).
 *   src_offsets:  host [n], byte offset of image i in d_src, a multiple of 16.
 *   heights, widths, channels: host [n]; channels 3 (RGB) or 4 (RGBA).
 *   out_dtype:    MIMO_F32 or MIMO_BF16.
 *   d_out:        device [out_rows_capacity, 1536] of out_dtype, 16-byte
 *                 aligned; rows [row_offsets[i], row_offsets[i+1]) belong
 *                 to image i, in the order of mimo_plan_batch.
 *   d_column_perm: device int32 [total_rows] or NULL. When given, receives
 *                 the column-order permutation of every image, as indices
 *                 into the whole batch (pixel_values[perm] works directly);
 *                 16-byte aligned; total_rows must fit int32
 *                 (MIMO_EOVERFLOW otherwise).
 * Every output row and permutation entry in [0, total_rows) is written
 * exactly once; nothing past total_rows is touched. Asynchronous on
 * `stream`; launch errors come back as MIMO_ECUDA.
 */
int mimo_preprocess_batch(const mimo_params *p, int32_t n,
                          const uint8_t *d_src, size_t src_bytes, const int64_t *src_offsets,
                          const int32_t *heights, const int32_t *widths, const int32_t *channels,
                          int32_t out_dtype, void *d_out, int64_t out_rows_capacity,
                          int32_t *d_column_perm, void *stream);

/*
 * Outputs of mimo_preprocess_batch_ex. Every pointer is a device pointer,
 * 16-byte aligned; the tables are optional (NULL = not written) and index the
 * whole batch, so they need total_rows to fit int32 (MIMO_EOVERFLOW).
 *   out_dtype, d_out, out_rows_capacity: as in mimo_preprocess_batch.
 *   row_order:      MIMO_ORDER_MERGE or MIMO_ORDER_COLUMN; only the position
 *                   of whole rows changes, never their contents.
 *   d_column_perm:  int32 [total_rows], perm[j] = merge-order row of the j-th
 *                   row in column order (column_permutation), whatever
 *                   row_order is.
 *   d_positions:    int32 [total_rows][2], (patch row, patch column) of every
 *                   emitted row in the image's patch grid: the 2-D rotary
 *                   positions of the vision tower (vision page,
 *                   MiMoVisionTransformer._rotary_positions), in the emitted
 *                   order.
 *   d_window_index: int32 [total_rows / 4], j-th entry = merge-order index of
 *                   the j-th merge unit in column-major order, batch-global
 *                   (vision page, MiMoVisionTransformer._get_window_index with
 *                   column_major; cortiq page, conventions).
 */
typedef struct {
    int32_t out_dtype;
    int32_t row_order;
    void *d_out;
    int64_t out_rows_capacity;
    int32_t *d_column_perm;
    int32_t *d_positions;
    int32_t *d_window_index;
} mimo_outputs;

/* The fused pixel path with the row order and the vision-tower index tables
 * chosen by `out`; all other arguments and guarantees as in
 * mimo_preprocess_batch (which is this call with merge order, no positions
 * and no window index). */
int mimo_preprocess_batch_ex(const mimo_params *p, int32_t n,
                             const uint8_t *d_src, size_t src_bytes, const int64_t *src_offsets,
                             const int32_t *heights, const int32_t *widths, const int32_t *channels,
                             const mimo_outputs *out, void *stream);

/*
 * A window of the batch's merge units, for splitting one batch (or one large
 * image) across devices by merge-block ranges. Merge unit u of the batch is
 * the 32x32 merge block whose 4 rows are batch rows 4u..4u+3 in merge order:
 * units are counted over the images in batch order, and inside an image in
 * merge-block order (block row, block col). The call runs the fused path of
 * mimo_preprocess_batch_ex on units [first_unit, first_unit + unit_count)
 * only, which may start and end inside an image.
 *   - Rows: merge order only (MIMO_ORDER_COLUMN -> MIMO_EUNSUPPORTED). d_out
 *     holds the window's rows: batch row 4u + k lands at row
 *     4 (u - first_unit) + k of d_out; out_rows_capacity >= 4 * unit_count.
 *     d_positions, if given, follows the rows the same way ([4 unit_count][2]).
 *   - d_column_perm [total_rows] and d_window_index [total_rows / 4] stay
 *     batch-global: the window writes the entries of its own units, at their
 *     batch positions and with batch-global values, and nothing else.
 *   - Windows that tile [0, total_rows / 4) write, between them, exactly what
 *     one mimo_preprocess_batch_ex call over the batch writes.
 * Errors: as mimo_preprocess_batch_ex; MIMO_EINVAL for a negative first_unit
 * or unit_count; MIMO_ERANGE when the window reaches past the batch's units.
 * An empty window launches nothing. Asynchronous on `stream`.
 */
int mimo_preprocess_units(const mimo_params *p, int32_t n,
                          const uint8_t *d_src, size_t src_bytes, const int64_t *src_offsets,
                          const int32_t *heights, const int32_t *widths, const int32_t *channels,
                          int64_t first_unit, int64_t unit_count, const mimo_outputs *out, void *stream);

/*
 * The same path from host memory to host memory (inputs copied in, rows and
 * permutation copied back), for callers whose images and results live on
 * the host. The caller supplies device staging buffers of at least the batch
 * size (d_src_stage >= src_bytes; d_out_stage >= total_rows rows of
 * out_dtype; d_perm_stage >= total_rows int32 when h_column_perm is not
 * NULL), so the call allocates nothing. Host buffers should be page-locked
 * for full copy bandwidth. The batch is cut into chunks of whole images (a
 * small first chunk, each later one three times larger, up to an eighth of
 * the batch) whose upload, kernel and download overlap on two library-created streams that
 * live only for the call, ordered after the work already on the caller's
 * stream. Synchronous: returns after the last copy to h_out has completed.
 */
int mimo_preprocess_batch_host(const mimo_params *p, int32_t n,
                               const uint8_t *h_src, size_t src_bytes, const int64_t *src_offsets,
                               const int32_t *heights, const int32_t *widths, const int32_t *channels,
                               int32_t out_dtype, void *h_out, int64_t out_rows_capacity,
                               int32_t *h_column_perm,
                               uint8_t *d_src_stage, size_t d_src_stage_bytes,
                               void *d_out_stage, int64_t d_out_stage_rows,
                               int32_t *d_perm_stage, void *stream);

/*
 * Host memory to host memory like mimo_preprocess_batch_host, for callers
 * that cannot allocate device memory (no cudaMalloc, no caching-allocator
 * call): images and rows are staged in a fixed area that the library itself
 * defines, MIMO_NOALLOC_STAGING_BYTES of device memory held by every GPU
 * that loads the library until the process exits. No counterpart on the
 * reference pages: it is an interface choice of this library.
 *   - Arguments and results are those of mimo_preprocess_batch_host without
 *     the three device staging buffers. The call runs on the current device;
 *     `stream` must belong to it. Synchronous: returns after the last copy
 *     to h_out has completed. A CUDA error part-way still waits for the
 *     work already queued on `stream` before it returns MIMO_ECUDA.
 *   - The batch is processed in chunks of whole images. An image whose
 *     uint8 bytes plus output rows (plus permutation entries when asked for)
 *     exceed the area, rounded up as the staging layout needs, is rejected
 *     with MIMO_ELIMIT before anything is copied or launched. With fp32 rows
 *     (24 bytes per resized pixel) an image of about 2.4 million resized
 *     pixels fits; a 1080x1920 RGBA image resized to 1088x1920 does.
 *   - Every call looks the area's device address up in the current
 *     device's context (cudaGetSymbolAddress), so a device reset or a new
 *     primary context never leaves a stale address behind. The first call on
 *     a device may load the library's device code there; make it before any
 *     stream capture.
 *   - Every call shares the one area and it keeps the last call's contents.
 *     Nothing in it needs to start at zero: each call writes every staged
 *     byte it reads. Calls that overlap on the GPU (from several host
 *     threads or streams at once) race on the area; serialise them.
 * Allocates no device or page-locked memory.
 */
#define MIMO_NOALLOC_STAGING_BYTES (64u << 20)
int mimo_preprocess_batch_host_noalloc(const mimo_params *p, int32_t n,
                                       const uint8_t *h_src, size_t src_bytes, const int64_t *src_offsets,
                                       const int32_t *heights, const int32_t *widths, const int32_t *channels,
                                       int32_t out_dtype, void *h_out, int64_t out_rows_capacity,
                                       int32_t *h_column_perm, void *stream);

/*
 * Prompt placeholder expansion (cortiq page, expand_prompt_ids): copies `ids`
 * to `out`, replacing the k-th occurrence of `pad_id` by counts[k] copies of
 * it. counts[k] is the number of vision tokens of the k-th media item:
 * mimo_num_patches / merge_size^2 for an image (get_number_of_image_patches
 * before the merge reduction, processing page). Host only.
 *   ids: host [n_ids]; counts: host [n_items], each >= 0; out: host
 *   [out_capacity]; *out_len receives the expanded length.
 * Errors: MIMO_EINVAL when the prompt holds a different number of
 * placeholders than n_items or a count is negative; MIMO_ECAPACITY when the
 * expansion does not fit out_capacity (nothing useful is left in out).
 */
int mimo_expand_prompt_ids(const int32_t *ids, int64_t n_ids, int32_t pad_id,
                           const int64_t *counts, int64_t n_items,
                           int32_t *out, int64_t out_capacity, int64_t *out_len);

/*
 * Video frames (cortiq page: prepare_video_frames, video_max_pixels,
 * smart_nframes, sample_frames). Decoding and frame selection from a file
 * stay with the caller; these take frames already decoded to HWC uint8.
 *
 * mimo_video_max_pixels: per-frame pixel ceiling for n sampled frames,
 *   max(min_pixels, min(total_max_pixels * temporal_patch_size // n,
 *   max_pixels)); total_max_pixels = 0 means no overall budget (max_pixels).
 * mimo_smart_nframes: the number of frames to sample: total / fps_src * fps,
 *   kept inside [min_frames, max_frames] and no larger than total, then
 *   rounded down to an even number; MIMO_EINVAL if that leaves 0.
 * mimo_sample_frames: idx = unique(int64(linspace(0, total - 1, n))) and
 *   ts = float32(idx) / fps_src; idx and ts hold n entries, *count gets the
 *   number of distinct indices written.
 * All three are host only.
 */
int mimo_video_max_pixels(int64_t n_sampled, int64_t total_max_pixels, const mimo_params *p, int64_t *out);
int mimo_smart_nframes(int64_t total, double fps_src, double fps, int64_t min_frames, int64_t max_frames,
                       int64_t *out);
int mimo_sample_frames(int64_t total, int64_t n, double fps_src, int64_t *idx, float *ts, int64_t *count);

/*
 * Plan of one video of n_frames frames of height x width: one smart_resize
 * under the per-frame budget for all frames, an odd count padded with its
 * last frame, grid_thw = (ceil(n/2), H'/16, W'/16), *rows = the product.
 * Host only.
 */
int mimo_plan_video(int32_t n_frames, int32_t height, int32_t width, int64_t total_max_pixels,
                    const mimo_params *p, int64_t *grid_thw, int64_t *rows);

/*
 * The pixel path for one video on the GPU. Frame f is at d_frames + f *
 * frame_stride (device, HWC uint8, all frames height x width x channels;
 * frame_stride a multiple of 16 and >= one frame's bytes; src_bytes covers
 * all frames, else MIMO_ERANGE). Consecutive frames pair up as temporal
 * patches: row (t, block row, block col, mh, mw), column (c, tt, py, px) takes
 * frame 2t + tt, the last frame standing in for a missing one. `out` as in
 * mimo_preprocess_batch_ex (the tables use the temporal patch t too: merge
 * units are listed per t). Asynchronous on `stream`.
 */
int mimo_preprocess_video(const mimo_params *p, int32_t n_frames, const uint8_t *d_frames, size_t src_bytes,
                          int64_t frame_stride, int32_t height, int32_t width, int32_t channels,
                          int64_t total_max_pixels, const mimo_outputs *out, void *stream);

/*
 * Patch embedding of the vision tower (vision page, MiMoVisionPatchEmbed: the
 * Conv3d with kernel = stride = (temporal 2, 16, 16) applied to the patch
 * rows) on the tensor cores:
 *   out[m, n] = sum_k rows[m, k] * weight[n, k] (+ bias[n]),  k < 1536,
 * with the weight laid out like the rows, (c, tt, py, px), i.e. the Conv3d
 * weight [embed_dim, 3, 2, 16, 16] flattened. bf16 inputs, fp32 accumulation.
 *   d_rows:   device bf16 [rows, 1536] (for example mimo_preprocess_batch with
 *             MIMO_BF16 output); rows >= 0.
 *   d_weight: device bf16 [embed_dim, 1536]; embed_dim a positive multiple
 *             of 256 (1280 for the MiMo-V2 tower).
 *   d_bias:   device fp32 [embed_dim] or NULL.
 *   d_out:    device [rows, embed_dim] of out_dtype (MIMO_F32 / MIMO_BF16).
 *   d_error:  device int32, read after the stream synchronises: 0, or a
 *             nonzero code if the kernel gave up waiting on its own pipeline
 *             (its output is then incomplete). The call does not clear it.
 * d_rows, d_weight, d_bias and d_out 16-byte aligned, d_error 4-byte aligned
 * (MIMO_EALIGN). An embed_dim that is not a positive multiple of 256 is
 * MIMO_EINVAL; rows above 2^31 - 1 is MIMO_EOVERFLOW (the tensor-map
 * coordinates are 32-bit). Asynchronous on `stream`.
 */
int mimo_patch_embed(const void *d_rows, int64_t rows, const void *d_weight, int32_t embed_dim,
                     const float *d_bias, int32_t out_dtype, void *d_out, int32_t *d_error, void *stream);

/*
 * Test hook for the failure path of mimo_patch_embed; no counterpart on the
 * pages. The same launch, except that the operand loaders of every CTA stop
 * after stop_after_kblocks 128-wide K blocks of its first tile (0 ..
 * 1536 / 128), so the tensor-core pipeline waits for operands that never
 * arrive, and each wait gives up after wait_rounds polling rounds (> 0)
 * instead of the default 2^20. The kernel then records a nonzero code in
 * *d_error (1: operands, 3: accumulator; the first role to give up wins),
 * stops every role, waits (bounded) for the copies and tensor-core work it
 * started, frees its tensor memory and returns; d_out is left incomplete.
 * Arguments otherwise as mimo_patch_embed (rows > 0). Asynchronous on
 * `stream`. For tests only: no normal call reaches this path.
 */
int mimo_patch_embed_stall_test(const void *d_rows, int64_t rows, const void *d_weight, int32_t embed_dim,
                                const float *d_bias, int32_t out_dtype, void *d_out, int32_t *d_error,
                                int32_t stop_after_kblocks, uint32_t wait_rounds, void *stream);

/*
 * The pixel path followed by the patch embedding, image run by image run
 * (vision page, MiMoVisionTransformer.forward: patch rows -> patch embed).
 * Images are grouped into runs whose bf16 patch rows fit half of d_scratch;
 * the runs alternate between the two halves. The pixel kernel writes a run's
 * rows on `stream`, and the patch-embedding GEMM (as mimo_patch_embed) reads
 * them on one of two streams the library keeps per host thread and device,
 * one per half, so it overlaps the next run's pixel kernel, and the next
 * run's GEMM can fill the SMs its last wave leaves idle. Events order each
 * GEMM after its rows and each reuse of a half after the GEMM that read it;
 * `stream` finally waits for both. Equal, bit for bit, to mimo_preprocess_batch_ex with
 * MIMO_BF16 rows followed by mimo_patch_embed on them.
 *   p, n, d_src, src_bytes, src_offsets, heights, widths, channels: as in
 *       mimo_preprocess_batch.
 *   row_order:  MIMO_ORDER_MERGE or MIMO_ORDER_COLUMN (order of the output rows).
 *   d_weight, embed_dim, d_bias, out_dtype, d_error: as in mimo_patch_embed.
 *   d_out:      device [total_rows, embed_dim] of out_dtype; out_rows_capacity
 *               its row count (MIMO_ECAPACITY if below total_rows).
 *   d_scratch:  device buffer of scratch_bytes, 16-byte aligned, owned by the
 *               caller; half of it must hold one image's rows (rows x 3072
 *               bytes), MIMO_ECAPACITY otherwise. About 2 x 96 MB or more
 *               keeps the GEMMs' last waves full. The rows are stored with an
 *               L2 evict-last policy and, once a GEMM has read a half, its
 *               lines are dropped from L2 without a write-back (when d_scratch
 *               is 128-byte aligned): its contents are undefined after the
 *               call. With halves of one image's rows (a 1080p image: 2 x 26 MB)
 *               the rows never reach HBM; larger halves trade that for fuller
 *               GEMM waves.
 * No permutation or index tables (mimo_preprocess_batch_ex writes those).
 * Asynchronous on `stream`. Argument errors return before anything is
 * queued; a CUDA error part-way waits for the library streams' queued GEMMs
 * before it returns, so none of them runs after the call.
 */
int mimo_preprocess_embed(const mimo_params *p, int32_t n, const uint8_t *d_src, size_t src_bytes,
                          const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                          const int32_t *channels, int32_t row_order, const void *d_weight, int32_t embed_dim,
                          const float *d_bias, int32_t out_dtype, void *d_out, int64_t out_rows_capacity,
                          void *d_scratch, size_t scratch_bytes, int32_t *d_error, void *stream);

/* Static description of a status code. */
const char *mimo_status_string(int status);

/* Library ABI version (major*10000 + minor*100 + patch). */
int mimo_version(void);

/*
 * Debug builds only (compiled with -DMIMO_BOUNDS_CHECK; no counterpart on the
 * pages): the number of accesses of the pixel kernels that failed their bounds
 * check since the last query, and the kind of the first (1: staged source copy
 * outside the caller's buffer, 2: direct source load outside the image, 3:
 * shared-memory tile index, 4: output row outside the validated rows, 5:
 * permutation / position / window entry outside its table). A failed check
 * skips its access and never traps. The query synchronises with the device's
 * earlier work and clears both values. Release builds return
 * MIMO_EUNSUPPORTED.
 */
int mimo_bounds_check_status(int64_t *violations, int32_t *first_kind);

#ifdef __cplusplus
}
#endif

#endif /* MIMO_H_ */
