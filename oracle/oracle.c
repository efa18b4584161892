/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of the MiMo-V2 image
 * preprocessing pixel path. It exists to check the CUDA library and nothing
 * else: only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg load it. The product library neither links nor calls it, and this file
 * includes none of the product's headers.
 *
 * What it follows (pages, by title and section):
 *   [P]  NeMo Automodel, "nemo_automodel.components.models.mimo_v2_flash.processing":
 *        module docstring (pixel path, sub-factor geometry contrast),
 *        class MimoV2ImageProcessor (order of the steps, default knobs),
 *        function _to_rgb (RGBA flattened onto white), function smart_resize
 *        (upscale branch, degenerate shrink rejected).
 *   [C]  docs.rs, "cortiq_engine::mimo_vision" module page: the bullet list of
 *        conventions (T = 2, (c, tt, py, px) rows, merge-block row order,
 *        column order), functions resize_bilinear, smart_resize and
 *        column_permutation.
 *   [V]  NeMo Automodel, "mimo_v2_flash.vision": MiMoVisionTransformer
 *        _rotary_positions and _get_window_index, MiMoVisionRotaryEmbedding.
 *        The pages give their signatures only; the tables here are the
 *        reading stated above each function (positions of the emitted rows;
 *        merge units in column-major order), pinned to hand-worked grids.
 *
 * Arithmetic: geometry in IEEE fp64 (as the Python original does), pixels in
 * fp64 from the uint8 values; every patch value is rounded to fp32 once, at
 * the very end. No blocking, fusion or reordering: each step is materialised
 * in full before the next one starts, in the order the processor page lists
 * them.
 *
 * Parity pins live in tests/test_oracle_*.py: closed forms, brute force,
 * invariants and library routines (transformers' Qwen2-VL smart_resize, PIL,
 * torch F.interpolate / conv3d, numpy). The one reading the pages leave open,
 * whether the long side scaled in the sub-factor upscale branch of
 * smart_resize is truncated to an integer, follows the MiMo-V2 processor of
 * the same serving lineage that is installed as a library (vLLM's MiMo-V2
 * Omni processor): it truncates, and the pins call it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_EINVAL 1      /* non-positive size, bad channel count, bad knob    */
#define OR_EASPECT 2     /* aspect ratio above 200 outside the upscale branch */
#define OR_EDEGENERATE 3 /* max_pixels shrink produced a zero side            */
#define OR_ECAPACITY 4   /* output buffer too small                           */
#define OR_ENOMEM 5

/* Python's round(): nearest integer, exact halves go to the even neighbour. */
static double py_round(double v)
{
    double lo = floor(v);
    double frac = v - lo;
    if (frac > 0.5)
        return lo + 1.0;
    if (frac < 0.5)
        return lo;
    return (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;
}

/*
 * [P] smart_resize / [C] smart_resize.
 * The HF (Qwen2-VL) smart_resize with two differences:
 *   - when the shorter side is under `factor`, both sides are first scaled by
 *     one ratio that brings it to exactly `factor`, and no aspect guard
 *     applies on that path;
 *   - when the max_pixels shrink floors a side to zero, that is an error
 *     rather than a value clamped up to `factor`.
 * HF algorithm as used here: aspect guard max/min > 200 is an error; round each
 * side to the nearest multiple of factor; if the area is above max_pixels,
 * shrink by beta = sqrt(h*w/max_pixels) and floor to the factor; else if the
 * area is below min_pixels, grow by beta = sqrt(min_pixels/(h*w)) and ceil.
 * The page names the sglang MiMoProcessor semantics for the upscale branch;
 * in that processor lineage the scaled long side is an integer, the float
 * quotient long*factor/short truncated (Python int()), and the later steps
 * run on the upscaled integer sizes.
 */
int oracle_smart_resize(int64_t height, int64_t width, int64_t factor,
                        int64_t min_pixels, int64_t max_pixels,
                        int64_t *out_h, int64_t *out_w)
{
    if (height <= 0 || width <= 0 || factor <= 0 || min_pixels < 0 || max_pixels <= 0)
        return OR_EINVAL;

    double h = (double)height;
    double w = (double)width;
    double f = (double)factor;

    if (height < factor || width < factor) {
        /* upscale branch: the short side becomes exactly `factor`, the long
           side the truncated quotient long * factor / short */
        if (height <= width) {
            w = trunc((double)(width * factor) / (double)height);
            h = f;
        } else {
            h = trunc((double)(height * factor) / (double)width);
            w = f;
        }
    } else {
        double big = h > w ? h : w;
        double small = h > w ? w : h;
        if (big / small > 200.0)
            return OR_EASPECT;
    }

    double h_bar = py_round(h / f) * f;
    double w_bar = py_round(w / f) * f;

    if (h_bar * w_bar > (double)max_pixels) {
        double beta = sqrt((h * w) / (double)max_pixels);
        h_bar = floor(h / beta / f) * f;
        w_bar = floor(w / beta / f) * f;
        if (h_bar == 0.0 || w_bar == 0.0)
            return OR_EDEGENERATE;
    } else if (h_bar * w_bar < (double)min_pixels) {
        double beta = sqrt((double)min_pixels / (h * w));
        h_bar = ceil(h * beta / f) * f;
        w_bar = ceil(w * beta / f) * f;
    }
    *out_h = (int64_t)h_bar;
    *out_w = (int64_t)w_bar;
    return OR_OK;
}

/*
 * [P] _to_rgb: an RGBA pixel is composited onto an opaque white background and
 * the result is an 8-bit RGB pixel. Exact value: c*a/255 + 255*(255-a)/255,
 * rounded to the nearest integer (255 is odd, so there are no ties).
 */
uint8_t oracle_flatten_on_white(uint8_t c, uint8_t a)
{
    int32_t num = (int32_t)c * (int32_t)a + 255 * (255 - (int32_t)a);
    /* nearest integer of num / 255 */
    return (uint8_t)((2 * num + 255) / 510);
}

/* [P] _to_rgb over a whole interleaved image: HWC uint8 (C = 3 or 4) -> HW3. */
int oracle_to_rgb(const uint8_t *src, int64_t H, int64_t W, int32_t C, uint8_t *rgb)
{
    if (C != 3 && C != 4)
        return OR_EINVAL;
    for (int64_t i = 0; i < H * W; ++i) {
        const uint8_t *px = src + i * C;
        for (int k = 0; k < 3; ++k)
            rgb[i * 3 + k] = (C == 4) ? oracle_flatten_on_white(px[k], px[3]) : px[k];
    }
    return OR_OK;
}

/* [P] _load: RGB uint8 -> planar float [3, H, W] on the 0..255 scale. */
void oracle_load_planes(const uint8_t *rgb, int64_t H, int64_t W, double *planes)
{
    for (int k = 0; k < 3; ++k)
        for (int64_t i = 0; i < H * W; ++i)
            planes[k * H * W + i] = (double)rgb[i * 3 + k];
}

/*
 * Source position of output index d along one axis, the align_corners=False
 * rule of torch.nn.functional.interpolate: src = (d + 0.5) * in/out - 0.5,
 * clamped at 0 from below; the two taps are floor(src) and the next index
 * (clamped to the last one), with weight lambda = src - floor(src) on the
 * second tap.
 */
static void axis_taps(int64_t d, int64_t in, int64_t out, int64_t *i0, int64_t *i1, double *lam)
{
    double scale = (double)in / (double)out;
    double src = ((double)d + 0.5) * scale - 0.5;
    if (src < 0.0)
        src = 0.0;
    int64_t lo = (int64_t)floor(src);
    *i0 = lo;
    *i1 = (lo + 1 < in) ? lo + 1 : in - 1;
    *lam = src - (double)lo;
}

/*
 * [P] class doc: F.interpolate(mode="bilinear", align_corners=False), no
 * antialias; [C] resize_bilinear: the same on a planar [c][h][w] image, taps
 * blended horizontally inside each of the two source rows, then those two
 * results blended vertically. No rounding back to 8 bits. One plane, fp64.
 */
void oracle_resize_plane(const double *in, int64_t in_h, int64_t in_w,
                         double *out, int64_t out_h, int64_t out_w)
{
    for (int64_t y = 0; y < out_h; ++y) {
        int64_t y0, y1;
        double ly;
        axis_taps(y, in_h, out_h, &y0, &y1, &ly);
        for (int64_t x = 0; x < out_w; ++x) {
            int64_t x0, x1;
            double lx;
            axis_taps(x, in_w, out_w, &x0, &x1, &lx);
            double top = (1.0 - lx) * in[y0 * in_w + x0] + lx * in[y0 * in_w + x1];
            double bot = (1.0 - lx) * in[y1 * in_w + x0] + lx * in[y1 * in_w + x1];
            out[y * out_w + x] = (1.0 - ly) * top + ly * bot;
        }
    }
}

/* [P] module docstring / class doc: standardise with mean and std expressed on
 * the 0..255 scale: (x - 255*mean_c) / (255*std_c). */
void oracle_normalize_planes(double *planes, int64_t HW, const double mean[3], const double stdv[3])
{
    for (int k = 0; k < 3; ++k) {
        double m = 255.0 * mean[k];
        double s = 255.0 * stdv[k];
        for (int64_t i = 0; i < HW; ++i)
            planes[k * HW + i] = (planes[k * HW + i] - m) / s;
    }
}

/*
 * [C] conventions, [P] class doc: one image stands for T identical frames
 * (T = temporal patch size). A patch row holds the values one Conv3d window
 * sees, in (c, tt, py, px) order, and the rows follow Qwen2-VL's merge-block
 * order (t, block row, block col, mh, mw).
 * planes: normalised [3, Hr, Wr]; out: [grid_t*grid_h*grid_w, 3*T*p*p] fp32.
 */
void oracle_patchify(const double *planes, int64_t Hr, int64_t Wr,
                     int32_t patch, int32_t temporal, int32_t merge, float *out)
{
    const int64_t p = patch, T = temporal, m = merge;
    const int64_t gh = Hr / p, gw = Wr / p;
    const int64_t gt = 1; /* one image = one temporal patch of T frames */
    const int64_t cols = 3 * T * p * p;
    int64_t row = 0;
    for (int64_t t = 0; t < gt; ++t)
        for (int64_t bh = 0; bh < gh / m; ++bh)
            for (int64_t bw = 0; bw < gw / m; ++bw)
                for (int64_t mh = 0; mh < m; ++mh)
                    for (int64_t mw = 0; mw < m; ++mw, ++row) {
                        int64_t col = 0;
                        for (int64_t c = 0; c < 3; ++c)
                            for (int64_t tt = 0; tt < T; ++tt) /* frame tt is a copy */
                                for (int64_t py = 0; py < p; ++py)
                                    for (int64_t px = 0; px < p; ++px, ++col) {
                                        int64_t y = (bh * m + mh) * p + py;
                                        int64_t x = (bw * m + mw) * p + px;
                                        out[row * cols + col] = (float)planes[c * Hr * Wr + y * Wr + x];
                                    }
                    }
}

/* Output rows of one image after smart_resize (gt*gh*gw), or -status. */
int64_t oracle_image_rows(int64_t H, int64_t W, int32_t patch, int32_t merge,
                          int64_t min_px, int64_t max_px)
{
    int64_t hr, wr;
    int st = oracle_smart_resize(H, W, (int64_t)patch * merge, min_px, max_px, &hr, &wr);
    if (st != OR_OK)
        return -(int64_t)st;
    return (hr / patch) * (wr / patch);
}

/*
 * [P] MimoV2ImageProcessor._process_one: the whole path for one image, step by
 * step: geometry, _to_rgb, _load, resize, standardise, duplicate + patchify.
 * grid_thw receives (1, Hr/patch, Wr/patch).
 */
int oracle_preprocess_image(const uint8_t *src, int64_t H, int64_t W, int32_t C,
                            int32_t patch, int32_t temporal, int32_t merge,
                            int64_t min_px, int64_t max_px,
                            const double mean[3], const double stdv[3],
                            float *out, int64_t out_rows_capacity, int64_t grid_thw[3])
{
    if (H <= 0 || W <= 0 || (C != 3 && C != 4) || patch <= 0 || temporal <= 0 || merge <= 0)
        return OR_EINVAL;
    int64_t Hr, Wr;
    int st = oracle_smart_resize(H, W, (int64_t)patch * merge, min_px, max_px, &Hr, &Wr);
    if (st != OR_OK)
        return st;
    const int64_t rows = (Hr / patch) * (Wr / patch);
    if (rows > out_rows_capacity)
        return OR_ECAPACITY;

    uint8_t *rgb = (uint8_t *)malloc((size_t)(H * W * 3));
    double *planes = (double *)malloc(sizeof(double) * (size_t)(3 * H * W));
    double *resized = (double *)malloc(sizeof(double) * (size_t)(3 * Hr * Wr));
    if (!rgb || !planes || !resized) {
        free(rgb);
        free(planes);
        free(resized);
        return OR_ENOMEM;
    }
    oracle_to_rgb(src, H, W, C, rgb);
    oracle_load_planes(rgb, H, W, planes);
    for (int k = 0; k < 3; ++k)
        oracle_resize_plane(planes + k * H * W, H, W, resized + k * Hr * Wr, Hr, Wr);
    oracle_normalize_planes(resized, Hr * Wr, mean, stdv);
    oracle_patchify(resized, Hr, Wr, patch, temporal, merge, out);

    grid_thw[0] = 1;
    grid_thw[1] = Hr / patch;
    grid_thw[2] = Wr / patch;
    free(rgb);
    free(planes);
    free(resized);
    return OR_OK;
}

/*
 * One patch value, evaluated directly from the definition for a single
 * (row, col) of one image's output (used to sample outputs of images too
 * large to run through oracle_preprocess_image in a test). Same steps, same
 * fp64 arithmetic, restricted to the four source pixels the value depends on.
 */
int oracle_patch_value(const uint8_t *src, int64_t H, int64_t W, int32_t C,
                       int64_t Hr, int64_t Wr, int32_t patch, int32_t temporal, int32_t merge,
                       const double mean[3], const double stdv[3],
                       int64_t row, int64_t col, float *value)
{
    const int64_t p = patch, T = temporal, m = merge;
    const int64_t gh = Hr / p, gw = Wr / p;
    if (row < 0 || row >= gh * gw || col < 0 || col >= 3 * T * p * p)
        return OR_EINVAL;
    /* row -> (block row, block col, mh, mw); col -> (c, tt, py, px) */
    int64_t unit = row / (m * m), sub = row % (m * m);
    int64_t bh = unit / (gw / m), bw = unit % (gw / m);
    int64_t mh = sub / m, mw = sub % m;
    int64_t px = col % p, py = (col / p) % p, c = col / (p * p * T);
    int64_t y = (bh * m + mh) * p + py;
    int64_t x = (bw * m + mw) * p + px;

    int64_t y0, y1, x0, x1;
    double ly, lx;
    axis_taps(y, H, Hr, &y0, &y1, &ly);
    axis_taps(x, W, Wr, &x0, &x1, &lx);
    double tap[2][2];
    int64_t ys[2] = {y0, y1}, xs[2] = {x0, x1};
    for (int a = 0; a < 2; ++a)
        for (int b = 0; b < 2; ++b) {
            const uint8_t *px_ = src + (ys[a] * W + xs[b]) * C;
            uint8_t v = (C == 4) ? oracle_flatten_on_white(px_[c], px_[3]) : px_[c];
            tap[a][b] = (double)v;
        }
    double top = (1.0 - lx) * tap[0][0] + lx * tap[0][1];
    double bot = (1.0 - lx) * tap[1][0] + lx * tap[1][1];
    double v = (1.0 - ly) * top + ly * bot;
    *value = (float)((v - 255.0 * mean[c]) / (255.0 * stdv[c]));
    return OR_OK;
}

/*
 * [C] column_permutation: the permutation that puts the rows into column
 * order. It visits merge units by (t, block col, block row) and keeps the m*m
 * rows of each unit adjacent and in their own order; perm[dst] = src.
 * Indices are offset by row0 (the image's first row in a batch), so they
 * index the concatenated batch directly.
 */
void oracle_column_permutation(int64_t grid_t, int64_t grid_h, int64_t grid_w,
                               int32_t merge, int64_t row0, int32_t *perm)
{
    const int64_t m = merge, gh2 = grid_h / m, gw2 = grid_w / m;
    int64_t dst = 0;
    for (int64_t t = 0; t < grid_t; ++t)
        for (int64_t b = 0; b < gw2; ++b)       /* block column */
            for (int64_t a = 0; a < gh2; ++a)   /* block row    */
                for (int64_t k = 0; k < m * m; ++k)
                    perm[dst++] = (int32_t)(row0 + ((t * gh2 + a) * gw2 + b) * m * m + k);
}

/*
 * [C] conventions, column order: the rows of oracle_patchify, with whole
 * merge units visited by (t, block col, block row) and the m*m rows of each
 * unit adjacent in (mh, mw) order. Equals the merge-order rows gathered with
 * oracle_column_permutation.
 */
void oracle_patchify_column(const double *planes, int64_t Hr, int64_t Wr,
                            int32_t patch, int32_t temporal, int32_t merge, float *out)
{
    const int64_t p = patch, T = temporal, m = merge;
    const int64_t gh = Hr / p, gw = Wr / p;
    const int64_t cols = 3 * T * p * p;
    int64_t row = 0;
    for (int64_t bw = 0; bw < gw / m; ++bw)
        for (int64_t bh = 0; bh < gh / m; ++bh)
            for (int64_t mh = 0; mh < m; ++mh)
                for (int64_t mw = 0; mw < m; ++mw, ++row) {
                    int64_t col = 0;
                    for (int64_t c = 0; c < 3; ++c)
                        for (int64_t tt = 0; tt < T; ++tt)
                            for (int64_t py = 0; py < p; ++py)
                                for (int64_t px = 0; px < p; ++px, ++col) {
                                    int64_t y = (bh * m + mh) * p + py;
                                    int64_t x = (bw * m + mw) * p + px;
                                    out[row * cols + col] = (float)planes[c * Hr * Wr + y * Wr + x];
                                }
                }
}

/*
 * Two-dimensional rotary positions of the vision tower (NeMo Automodel
 * "mimo_v2_flash.vision", MiMoVisionTransformer._rotary_positions and
 * MiMoVisionRotaryEmbedding: two-dimensional frequencies): for every patch
 * row, its patch row index and patch column index in the grid, in the order
 * the rows are emitted (merge-block order, or column order when
 * column_order != 0: [C] conventions, the rotary tables follow the rows'
 * permutation). pos has 2 entries per row: (h, w).
 */
void oracle_rotary_positions(int64_t grid_t, int64_t grid_h, int64_t grid_w, int32_t merge,
                             int32_t column_order, int32_t *pos)
{
    const int64_t m = merge, gh2 = grid_h / m, gw2 = grid_w / m;
    int64_t row = 0;
    for (int64_t t = 0; t < grid_t; ++t)
        for (int64_t a = 0; a < (column_order ? gw2 : gh2); ++a)
            for (int64_t b = 0; b < (column_order ? gh2 : gw2); ++b)
                for (int64_t mh = 0; mh < m; ++mh)
                    for (int64_t mw = 0; mw < m; ++mw, ++row) {
                        int64_t bh = column_order ? b : a;
                        int64_t bw = column_order ? a : b;
                        pos[2 * row + 0] = (int32_t)(bh * m + mh);
                        pos[2 * row + 1] = (int32_t)(bw * m + mw);
                    }
}

/*
 * Window index over merge units (MiMoVisionTransformer._get_window_index with
 * column_major; [C] conventions: column-order windows list whole merge units
 * by (t, block col, block row)): win[j] = merge-order index of the j-th unit
 * in column-major order, offset by unit0 (the image's first unit in a batch).
 */
void oracle_window_index(int64_t grid_t, int64_t grid_h, int64_t grid_w, int32_t merge,
                         int64_t unit0, int32_t *win)
{
    const int64_t m = merge, gh2 = grid_h / m, gw2 = grid_w / m;
    int64_t j = 0;
    for (int64_t t = 0; t < grid_t; ++t)
        for (int64_t b = 0; b < gw2; ++b)
            for (int64_t a = 0; a < gh2; ++a)
                win[j++] = (int32_t)(unit0 + (t * gh2 + a) * gw2 + b);
}

/*
 * [C] expand_prompt_ids: each media placeholder token of the rendered prompt
 * is expanded into as many copies as the media item has vision tokens (for an
 * image: grid_h * grid_w / merge^2, [P] get_number_of_image_patches divided
 * by the merge reduction). Placeholders are matched to items in order.
 * Returns the expanded length, or -1 if the prompt holds a different number
 * of placeholders than items, or -2 if out_capacity is too small.
 */
int64_t oracle_expand_prompt_ids(const int32_t *ids, int64_t n_ids, int32_t pad_id,
                                 const int64_t *counts, int64_t n_items,
                                 int32_t *out, int64_t out_capacity)
{
    int64_t used = 0, len = 0;
    for (int64_t i = 0; i < n_ids; ++i) {
        if (ids[i] == pad_id) {
            if (used >= n_items)
                return -1;
            for (int64_t k = 0; k < counts[used]; ++k) {
                if (len >= out_capacity)
                    return -2;
                out[len++] = pad_id;
            }
            ++used;
        } else {
            if (len >= out_capacity)
                return -2;
            out[len++] = ids[i];
        }
    }
    return used == n_items ? len : -1;
}

/* ------------------------------------------------------------------ video */

/*
 * [C] video_max_pixels: per-frame pixel ceiling for n sampled frames,
 * max(min_pixels, min(total_max * T // n, max_pixels)).
 */
int64_t oracle_video_max_pixels(int64_t n_sampled, int64_t total_max, int32_t temporal,
                                int64_t min_pixels, int64_t max_pixels)
{
    int64_t share = (total_max * temporal) / n_sampled; /* floor division, all >= 0 */
    int64_t cap = share < max_pixels ? share : max_pixels;
    return cap > min_pixels ? cap : min_pixels;
}

/*
 * [C] smart_nframes: the number of frames to sample. Start from
 * total / fps_src * fps, keep it inside [min_frames, max_frames] and no
 * larger than total, then round it down to an even number. A result of 0
 * frames is an error (OR_EINVAL), as is a non-positive count or rate.
 */
int oracle_smart_nframes(int64_t total, double fps_src, double fps, int64_t min_frames, int64_t max_frames,
                         int64_t *out)
{
    if (total <= 0 || !(fps_src > 0.0) || !(fps > 0.0) || min_frames < 0 || max_frames < min_frames)
        return OR_EINVAL;
    double n = (double)total / fps_src * fps;
    if (n < (double)min_frames)
        n = (double)min_frames;
    if (n > (double)max_frames)
        n = (double)max_frames;
    if (n > (double)total)
        n = (double)total;
    int64_t even = (int64_t)floor(n / 2.0) * 2;
    if (even <= 0)
        return OR_EINVAL;
    *out = even;
    return OR_OK;
}

/*
 * [C] sample_frames: indices unique(int64(linspace(0, total - 1, n))) and
 * timestamps float32(idx) / fps_src. linspace: start + k * (stop - start) /
 * (n - 1) in fp64 with the last sample exactly stop (n = 1 gives [0]); int64
 * truncates; unique keeps one of each value in increasing order. Returns the
 * number of indices written (<= n), or -1 on bad arguments.
 */
int64_t oracle_sample_frames(int64_t total, int64_t n, double fps_src, int64_t *idx, float *ts)
{
    if (total <= 0 || n <= 0 || !(fps_src > 0.0))
        return -1;
    double stop = (double)(total - 1);
    double step = n > 1 ? stop / (double)(n - 1) : 0.0;
    int64_t count = 0;
    for (int64_t k = 0; k < n; ++k) {
        double v = (k == n - 1 && n > 1) ? stop : (double)k * step;
        int64_t i = (int64_t)v;
        if (count > 0 && idx[count - 1] == i)
            continue; /* linspace is non-decreasing: duplicates are adjacent */
        idx[count] = i;
        ts[count] = (float)i / (float)fps_src;
        ++count;
    }
    return count;
}

/*
 * [C] prepare_video_frames, pixel part: frames (HWC uint8, all H x W x C, at
 * stride `frame_stride` bytes) -> per-frame budget video_max_pixels(n, ...),
 * one smart_resize for all frames, an odd count padded by repeating the last
 * frame, each frame through _to_rgb, _load, resize and standardisation, and
 * consecutive frames paired as temporal patches: row (t, block row, block
 * col, mh, mw), column (c, tt, py, px) taking frame 2t + tt.
 * total_max <= 0 means no budget (max_pixels applies as it is).
 */
int oracle_preprocess_video(const uint8_t *frames, int64_t n, int64_t frame_stride, int64_t H, int64_t W,
                            int32_t C, int32_t patch, int32_t temporal, int32_t merge,
                            int64_t min_px, int64_t max_px, int64_t total_max,
                            const double mean[3], const double stdv[3],
                            float *out, int64_t out_rows_capacity, int64_t grid_thw[3])
{
    if (n <= 0 || H <= 0 || W <= 0 || (C != 3 && C != 4) || temporal != 2)
        return OR_EINVAL;
    const int64_t budget = total_max > 0 ? oracle_video_max_pixels(n, total_max, temporal, min_px, max_px) : max_px;
    int64_t Hr, Wr;
    int st = oracle_smart_resize(H, W, (int64_t)patch * merge, min_px, budget, &Hr, &Wr);
    if (st != OR_OK)
        return st;
    const int64_t n_pad = n + (n & 1);
    const int64_t gt = n_pad / 2, gh = Hr / patch, gw = Wr / patch;
    if (gt * gh * gw > out_rows_capacity)
        return OR_ECAPACITY;

    uint8_t *rgb = (uint8_t *)malloc((size_t)(H * W * 3));
    double *planes = (double *)malloc(sizeof(double) * (size_t)(3 * H * W));
    double *resized = (double *)malloc(sizeof(double) * (size_t)(n * 3 * Hr * Wr));
    if (!rgb || !planes || !resized) {
        free(rgb);
        free(planes);
        free(resized);
        return OR_ENOMEM;
    }
    for (int64_t f = 0; f < n; ++f) {
        double *r = resized + f * 3 * Hr * Wr;
        oracle_to_rgb(frames + f * frame_stride, H, W, C, rgb);
        oracle_load_planes(rgb, H, W, planes);
        for (int k = 0; k < 3; ++k)
            oracle_resize_plane(planes + k * H * W, H, W, r + k * Hr * Wr, Hr, Wr);
        oracle_normalize_planes(r, Hr * Wr, mean, stdv);
    }
    const int64_t p = patch, T = temporal, m = merge, cols = 3 * T * p * p;
    int64_t row = 0;
    for (int64_t t = 0; t < gt; ++t)
        for (int64_t bh = 0; bh < gh / m; ++bh)
            for (int64_t bw = 0; bw < gw / m; ++bw)
                for (int64_t mh = 0; mh < m; ++mh)
                    for (int64_t mw = 0; mw < m; ++mw, ++row) {
                        int64_t col = 0;
                        for (int64_t c = 0; c < 3; ++c)
                            for (int64_t tt = 0; tt < T; ++tt) {
                                int64_t f = t * T + tt;
                                if (f > n - 1)
                                    f = n - 1; /* an odd count reuses its final frame */
                                const double *pl = resized + f * 3 * Hr * Wr + c * Hr * Wr;
                                for (int64_t py = 0; py < p; ++py)
                                    for (int64_t px = 0; px < p; ++px, ++col) {
                                        int64_t y = (bh * m + mh) * p + py;
                                        int64_t x = (bw * m + mw) * p + px;
                                        out[row * cols + col] = (float)pl[y * Wr + x];
                                    }
                            }
                    }
    grid_thw[0] = gt;
    grid_thw[1] = gh;
    grid_thw[2] = gw;
    free(rgb);
    free(planes);
    free(resized);
    return OR_OK;
}

/*
 * [V] MiMoVisionPatchEmbed: the Conv3d with kernel = stride = (T, p, p) over
 * the frames is, for each patch row, the dot product of the row's 3*T*p*p
 * values (c, tt, py, px) with each output channel's weight of the same layout:
 * out[m][n] = sum_k rows[m][k] * w[n][k] (+ bias[n]), in fp64.
 */
void oracle_patch_embed(const float *rows, int64_t M, int64_t K, const float *w, int64_t N,
                        const double *bias, double *out)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = bias ? bias[n] : 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)rows[m * K + k] * (double)w[n * K + k];
            out[m * N + n] = acc;
        }
}
