// mimo_api.cpp -- host side of the C ABI declared in include/mimo.h:
// geometry (smart_resize), batch planning, argument validation, per-launch
// descriptor blocks and the host-memory pipeline. All pixel work happens in
// the CUDA kernel (mimo_preprocess.cu).
#include "mimo.h"

#include <cuda_runtime_api.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstring>
#include <limits>
#include <vector>

#include "mimo_internal.h"

namespace {

constexpr int64_t kFactor = mimo::kBlock;  // patch 16 x merge 2

// NVTX range around a host step (plan, upload, kernel launch, download, wait), so
// that a timeline profiler shows where a call spends its host time. Without an
// attached tool a push/pop is a check of one function pointer.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

bool supported_knobs(const mimo_params *p) {
    return p->patch_size == 16 && p->temporal_patch_size == 2 && p->merge_size == 2 && p->reserved == 0;
}

int check_params(const mimo_params *p) {
    if (!p) return MIMO_EINVAL;
    if (p->min_pixels < 0 || p->max_pixels <= 0) return MIMO_EINVAL;
    if (!supported_knobs(p)) return MIMO_EUNSUPPORTED;
    for (int c = 0; c < 3; ++c) {
        if (!std::isfinite(p->image_mean[c]) || !std::isfinite(p->image_std[c]) || !(p->image_std[c] > 0.f))
            return MIMO_EUNSUPPORTED;
    }
    return MIMO_OK;
}

// Nearest integer with ties to even (the default IEEE rounding mode), the
// behaviour of Python's round() on the processor's float quotients.
double round_ties_even(double v) {
    const int saved = std::fegetround();
    if (saved != FE_TONEAREST) std::fesetround(FE_TONEAREST);
    const double r = std::nearbyint(v);
    if (saved != FE_TONEAREST) std::fesetround(saved);
    return r;
}

// smart_resize of the processing page: sub-factor upscale first (no aspect
// guard in that branch), else the HF aspect guard; round to the factor; then
// the max_pixels shrink (floor, zero side rejected) or min_pixels growth (ceil).
// In the upscale branch the long side becomes the integer part of
// long * factor / short, as the MiMo processor lineage the page names (sglang
// MiMoProcessor semantics) computes it; the later steps use those integer sizes.
int smart_resize_impl(int64_t height, int64_t width, int64_t factor, int64_t min_px, int64_t max_px,
                      int64_t *oh, int64_t *ow) {
    if (height <= 0 || width <= 0 || factor <= 0 || min_px < 0 || max_px <= 0 || !oh || !ow) return MIMO_EINVAL;
    // sizes whose products could overflow the exact-integer steps below
    const int64_t lim = int64_t(1) << 31;
    if (height >= lim || width >= lim || factor >= lim) return MIMO_EOVERFLOW;

    const double f = static_cast<double>(factor);
    double h, w;
    const int64_t short_side = std::min(height, width);
    if (short_side < factor) {
        // both sides scaled by factor/short: the short side lands exactly on the
        // factor, the long side on the floor of the exact quotient (both operands
        // are positive and below 2^31, so the product is exact in 64 bits)
        if (height == short_side) {
            h = f;
            w = static_cast<double>((width * factor) / height);
        } else {
            w = f;
            h = static_cast<double>((height * factor) / width);
        }
    } else {
        const double ratio = static_cast<double>(std::max(height, width)) / static_cast<double>(short_side);
        if (ratio > 200.0) return MIMO_EASPECT;
        h = static_cast<double>(height);
        w = static_cast<double>(width);
    }

    double hb = round_ties_even(h / f) * f;
    double wb = round_ties_even(w / f) * f;
    const double area = hb * wb;
    if (area > static_cast<double>(max_px)) {
        const double beta = std::sqrt((h * w) / static_cast<double>(max_px));
        hb = std::floor(h / beta / f) * f;
        wb = std::floor(w / beta / f) * f;
        if (hb <= 0.0 || wb <= 0.0) return MIMO_EDEGENERATE;
    } else if (area < static_cast<double>(min_px)) {
        const double beta = std::sqrt(static_cast<double>(min_px) / (h * w));
        hb = std::ceil(h * beta / f) * f;
        wb = std::ceil(w * beta / f) * f;
    }
    if (hb > 9.0e15 || wb > 9.0e15) return MIMO_EOVERFLOW;
    *oh = static_cast<int64_t>(hb);
    *ow = static_cast<int64_t>(wb);
    return MIMO_OK;
}

// Geometry of one image for the kernel, or a status.
struct ImagePlan {
    int64_t Hr, Wr, rows, blocks;
    int32_t flags;
    int32_t tile_rows, tile_cols;
};

int64_t axis_max_span(int64_t in, int64_t out) {
    int64_t span = 0;
    for (int64_t b = 0; b < out / mimo::kBlock; ++b) span = std::max(span, mimo::block_span(b, in, out));
    return span;
}

int plan_image(int64_t H, int64_t W, const mimo_params *p, ImagePlan *ip) {
    int64_t Hr = 0, Wr = 0;
    const int st = smart_resize_impl(H, W, kFactor, p->min_pixels, p->max_pixels, &Hr, &Wr);
    if (st != MIMO_OK) return st;
    // the kernel's tap arithmetic keeps 2 * (resized side) in 32 bits; a side of
    // 2^30 would mean hundreds of GB of rows anyway
    if (Hr >= (int64_t(1) << 30) || Wr >= (int64_t(1) << 30)) return MIMO_EOVERFLOW;
    ip->Hr = Hr;
    ip->Wr = Wr;
    ip->rows = (Hr / 16) * (Wr / 16);
    ip->blocks = (Hr / mimo::kBlock) * (Wr / mimo::kBlock);
    if (ip->blocks > INT32_MAX / 2) return MIMO_EOVERFLOW;
    ip->flags = 0;
    // rows
    if (Hr == H) {
        ip->flags |= mimo::kIdentityRows;  // every weight is 0: only the first tap is staged
        ip->tile_rows = mimo::kBlock;
    } else {
        const int64_t rs = axis_max_span(H, Hr);
        if (rs > mimo::kMaxTile) {
            ip->flags |= mimo::kGatherRows;
            ip->tile_rows = mimo::kMaxTile;
        } else {
            ip->tile_rows = static_cast<int32_t>(rs);
        }
    }
    // columns
    if (Wr == W) {
        ip->flags |= mimo::kIdentityCols;
        ip->tile_cols = mimo::kBlock;
    } else {
        const int64_t cs = axis_max_span(W, Wr);
        if (cs > mimo::kMaxTile) {
            ip->flags |= mimo::kGatherCols;
            ip->tile_cols = mimo::kMaxTile;
        } else {
            ip->tile_cols = static_cast<int32_t>(cs);
        }
    }
    return MIMO_OK;
}

struct BatchPlan {
    std::vector<ImagePlan> img;
    std::vector<int64_t> row0;  // n + 1
};

int plan_all(int32_t n, const int32_t *heights, const int32_t *widths, const mimo_params *p, BatchPlan *bp) {
    NvtxRange range("mimo plan");
    bp->img.resize(static_cast<size_t>(n));
    bp->row0.assign(static_cast<size_t>(n) + 1, 0);
    for (int32_t i = 0; i < n; ++i) {
        if (heights[i] <= 0 || widths[i] <= 0) return MIMO_EINVAL;
        const int st = plan_image(heights[i], widths[i], p, &bp->img[i]);
        if (st != MIMO_OK) return st;
        if (bp->row0[i] > std::numeric_limits<int64_t>::max() / 2) return MIMO_EOVERFLOW;
        bp->row0[i + 1] = bp->row0[i] + bp->img[i].rows;
    }
    return MIMO_OK;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

struct Validated {
    BatchPlan plan;
    int64_t total_rows = 0;
};

// Shared argument checks of the two batch entry points (device or host
// buffers); `src`/`out`/`perm` are whatever the call will read and write.
int validate_batch(const mimo_params *p, int32_t n, const void *src, size_t src_bytes, const int64_t *src_offsets,
                   const int32_t *heights, const int32_t *widths, const int32_t *channels, int32_t out_dtype,
                   const void *out, int64_t out_rows_capacity, const void *perm, Validated *v) {
    int st = check_params(p);
    if (st != MIMO_OK) return st;
    if (n < 0) return MIMO_EINVAL;
    if (out_dtype != MIMO_F32 && out_dtype != MIMO_BF16) return MIMO_EINVAL;
    if (n == 0) return MIMO_OK;
    if (!src || !src_offsets || !heights || !widths || !channels) return MIMO_EINVAL;
    for (int32_t i = 0; i < n; ++i) {
        if (channels[i] != 3 && channels[i] != 4) return MIMO_ECHANNELS;
        if (src_offsets[i] < 0) return MIMO_EINVAL;
        if ((src_offsets[i] & 15) != 0) return MIMO_EALIGN;
    }
    if (!aligned16(src)) return MIMO_EALIGN;
    st = plan_all(n, heights, widths, p, &v->plan);
    if (st != MIMO_OK) return st;
    for (int32_t i = 0; i < n; ++i) {
        const uint64_t bytes = static_cast<uint64_t>(heights[i]) * static_cast<uint64_t>(widths[i]) *
                               static_cast<uint64_t>(channels[i]);
        const uint64_t off = static_cast<uint64_t>(src_offsets[i]);
        if (off > src_bytes || bytes > src_bytes - off) return MIMO_ERANGE;
    }
    v->total_rows = v->plan.row0[n];
    if (v->total_rows > out_rows_capacity) return MIMO_ECAPACITY;
    if (!out) return MIMO_EINVAL;
    if (!aligned16(out)) return MIMO_EALIGN;
    if (perm) {
        if (!aligned16(perm)) return MIMO_EALIGN;
        if (v->total_rows > INT32_MAX) return MIMO_EOVERFLOW;
    }
    return MIMO_OK;
}

void fold_normalisation(const mimo_params *p, mimo::LaunchParams *lp) {
    for (int c = 0; c < 3; ++c) {
        const double s = 255.0 * static_cast<double>(p->image_std[c]);
        const double m = 255.0 * static_cast<double>(p->image_mean[c]);
        lp->k[c] = static_cast<float>(1.0 / s);
        lp->b[c] = static_cast<float>(-m / s);
    }
}

// Launches images [first, last) of a validated batch, cut into launches of at
// most kMaxImagesPerLaunch images and INT32_MAX blocks. Output rows and
// source offsets stay batch-global.
struct Tables {
    int32_t order = MIMO_ORDER_MERGE;
    int32_t *pos = nullptr;
    int32_t *win = nullptr;
};

// A window of merge units: units [lo, hi) of the batch, counted over the images
// in batch order and in merge order inside each image (unit u holds batch rows
// 4u..4u+3 in merge order). Emitted rows (and their rotary positions) land
// `row_shift` rows before their batch row; the permutation and the window
// index stay batch-global.
struct UnitWindow {
    int64_t lo = 0, hi = std::numeric_limits<int64_t>::max();
    int64_t row_shift = 0;
};

int launch_range(const mimo_params *p, const Validated &v, int32_t first, int32_t last, const uint8_t *d_src,
                 size_t src_bytes, const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                 const int32_t *channels, int32_t out_dtype, void *d_out, int32_t *d_perm, void *stream,
                 const Tables &tables = Tables(), int64_t row_base = 0, const UnitWindow &win = UnitWindow(),
                 bool keep_rows = false) {
    NvtxRange range("mimo launch");
    static thread_local mimo::LaunchParams lp;  // 31 KB: kept off the stack
    // units of image i inside the window: [lo_i, hi_i) of its own units
    auto unit_span = [&](int32_t i, int64_t *lo_i, int64_t *hi_i) {
        const int64_t u0 = v.plan.row0[i] / 4;
        *lo_i = std::max<int64_t>(win.lo - u0, 0);
        *hi_i = std::min<int64_t>(win.hi - u0, v.plan.img[i].blocks);
        return *hi_i > *lo_i;
    };
    // emitted rows land row_shift rows early: shift the row and position bases (addresses only; every
    // row the window writes lies at or after row_shift)
    const uintptr_t out_base = reinterpret_cast<uintptr_t>(d_out) -
                               static_cast<uintptr_t>(win.row_shift) * mimo::kRowWidth * (out_dtype == MIMO_BF16 ? 2u : 4u);
    const uintptr_t pos_base = reinterpret_cast<uintptr_t>(tables.pos) -
                               static_cast<uintptr_t>(win.row_shift) * 2u * sizeof(int32_t);
    int32_t i = first;
    int64_t lo_i = 0, hi_i = 0;
    while (i < last && !unit_span(i, &lo_i, &hi_i)) ++i;
    while (i < last) {
        std::memset(&lp, 0, sizeof(lp));
        lp.src = d_src;
        lp.out = reinterpret_cast<void *>(out_base);
        lp.perm = d_perm;
        lp.pos = tables.pos ? reinterpret_cast<int32_t *>(pos_base) : nullptr;
        lp.win = tables.win;
        lp.order = tables.order;
        lp.unit0 = static_cast<int32_t>(lo_i);  // the launch's first image may start inside it
        lp.keep_rows = keep_rows ? 1 : 0;
        fold_normalisation(p, &lp);
        int64_t blocks = 0;
        int32_t tr = 1, tc = 1, k = 0;
        int64_t wr = 1, wc = 1;  // warp-staged kernel: source rows per warp, source columns per block
        while (i < last && k < mimo::kMaxImagesPerLaunch && blocks + (hi_i - lo_i) <= static_cast<int64_t>(INT32_MAX)) {
            const ImagePlan &ip = v.plan.img[i];
            mimo::ImageDesc &d = lp.img[k];
            d.src_off = src_offsets[i];
            d.row0 = v.plan.row0[i] - row_base;  // rows land at d_out + (row0 - row_base) * 1536
            d.H = heights[i];
            d.W = widths[i];
            d.Hr = static_cast<int32_t>(ip.Hr);
            d.Wr = static_cast<int32_t>(ip.Wr);
            d.flags = ip.flags | (channels[i] << mimo::kChannelShift);
            d.frame_stride = 0;
            d.frames = 1;
            // staging copies are 16-byte chunks that may run up to 15 bytes past
            // the image; they read nothing past the end of the caller's buffer
            d.limit = static_cast<int64_t>(src_bytes) - src_offsets[i];
            lp.block_start[k] = static_cast<int32_t>(blocks);
            blocks += hi_i - lo_i;
            tr = std::max(tr, ip.tile_rows);
            // the taps of 4 consecutive output rows span at most floor(3 H / Hr) + 3 source rows,
            // those of 32 consecutive columns at most floor(31 W / Wr) + 3 source columns
            wr = std::max<int64_t>(wr, 3 * static_cast<int64_t>(heights[i]) / ip.Hr + 3);
            wc = std::max<int64_t>(wc, 31 * static_cast<int64_t>(widths[i]) / ip.Wr + 3);
            tc = std::max(tc, ip.tile_cols);
            ++k;
            // the next image with units in the window; only the window's first image starts inside
            // itself, so later images of a launch begin at their unit 0
            do {
                ++i;
            } while (i < last && !unit_span(i, &lo_i, &hi_i));
        }
        lp.block_start[k] = static_cast<int32_t>(blocks);
        lp.n = k;
        lp.tile_rows = tr;
        // 16-byte rows (whole-float4 staging stores and loads), at least the 32
        // columns the in-place horizontal pass writes
        lp.tile_stride = (std::max(tc, mimo::kBlock) + 3) & ~3;
        const size_t tile_floats = 3u * static_cast<size_t>(tr) * static_cast<size_t>(lp.tile_stride);
        // raw staging rows: a row segment of up to 4*tc bytes at any 16-byte
        // misalignment, plus the word a 12-byte RGB read may touch past it
        lp.raw_stride = ((32 + 4 * tc) + 15) & ~15;
        const size_t raw_floats = static_cast<size_t>(tr) * static_cast<size_t>(lp.raw_stride) / 4u;
        lp.raw = static_cast<int32_t>(tile_floats);  // tile | raw staging rows
        const size_t smem = sizeof(float) * (tile_floats + raw_floats);
        // warp-staged kernel (launches that gather no axis): a row segment of up to 4 * wc bytes at any
        // 16-byte misalignment, plus the word a 12-byte RGB read may touch past it
        lp.warp_rows = static_cast<int32_t>(std::min<int64_t>(wr, INT32_MAX));
        lp.warp_stride = static_cast<int32_t>(((32 + 4 * std::min<int64_t>(wc, 1 << 20)) + 15) & ~int64_t(15));
#if defined(MIMO_BOUNDS_CHECK)
        // rows this call may emit (kernel numbering: batch row - row_base), inside the window
        lp.chk_row_lo = std::max<int64_t>(v.plan.row0[first], 4 * win.lo) - row_base;
        lp.chk_row_hi = std::min<int64_t>(v.plan.row0[last], win.hi > INT64_MAX / 4 ? INT64_MAX : 4 * win.hi) - row_base;
        lp.chk_table_rows = v.plan.row0[last] - row_base;
        lp.chk_smem_floats = static_cast<int32_t>(tile_floats + raw_floats);
#endif
        const int st = mimo::launch_preprocess(lp, blocks, out_dtype, smem, stream);
        if (st != MIMO_OK) return st;
    }
    return MIMO_OK;
}

size_t dtype_bytes(int32_t out_dtype) { return out_dtype == MIMO_BF16 ? 2u : 4u; }

}  // namespace

extern "C" {

void mimo_params_default(mimo_params *p) {
    if (!p) return;
    std::memset(p, 0, sizeof(*p));
    p->patch_size = 16;
    p->temporal_patch_size = 2;
    p->merge_size = 2;
    p->min_pixels = 8192;
    p->max_pixels = 8388608;
    const float mean[3] = {0.485f, 0.456f, 0.406f};
    const float stdv[3] = {0.229f, 0.224f, 0.225f};
    for (int c = 0; c < 3; ++c) {
        p->image_mean[c] = mean[c];
        p->image_std[c] = stdv[c];
    }
}

int mimo_smart_resize(int64_t height, int64_t width, int64_t factor, int64_t min_pixels, int64_t max_pixels,
                      int64_t *out_height, int64_t *out_width) {
    return smart_resize_impl(height, width, factor, min_pixels, max_pixels, out_height, out_width);
}

int mimo_num_patches(int64_t height, int64_t width, const mimo_params *p, int64_t *out_patches) {
    if (!p || !out_patches) return MIMO_EINVAL;
    if (p->patch_size <= 0 || p->merge_size <= 0) return MIMO_EINVAL;
    int64_t oh = 0, ow = 0;
    const int64_t factor = static_cast<int64_t>(p->patch_size) * p->merge_size;
    const int st = smart_resize_impl(height, width, factor, p->min_pixels, p->max_pixels, &oh, &ow);
    if (st != MIMO_OK) return st;
    *out_patches = (oh / p->patch_size) * (ow / p->patch_size);
    return MIMO_OK;
}

int mimo_plan_batch(int32_t n, const int32_t *heights, const int32_t *widths, const mimo_params *p,
                    int64_t *grid_thw, int64_t *row_offsets) {
    const int st0 = check_params(p);
    if (st0 != MIMO_OK) return st0;
    if (n < 0 || !row_offsets) return MIMO_EINVAL;
    if (n > 0 && (!heights || !widths || !grid_thw)) return MIMO_EINVAL;
    BatchPlan bp;
    const int st = plan_all(n, heights, widths, p, &bp);
    if (st != MIMO_OK) return st;
    for (int32_t i = 0; i < n; ++i) {
        grid_thw[3 * i + 0] = 1;
        grid_thw[3 * i + 1] = bp.img[i].Hr / 16;
        grid_thw[3 * i + 2] = bp.img[i].Wr / 16;
    }
    std::memcpy(row_offsets, bp.row0.data(), sizeof(int64_t) * (static_cast<size_t>(n) + 1));
    return MIMO_OK;
}

int mimo_preprocess_batch_ex(const mimo_params *p, int32_t n, const uint8_t *d_src, size_t src_bytes,
                             const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                             const int32_t *channels, const mimo_outputs *out, void *stream) {
    if (!out) return MIMO_EINVAL;
    if (out->row_order != MIMO_ORDER_MERGE && out->row_order != MIMO_ORDER_COLUMN) return MIMO_EINVAL;
    Validated v;
    int st = validate_batch(p, n, d_src, src_bytes, src_offsets, heights, widths, channels, out->out_dtype,
                            out->d_out, out->out_rows_capacity, out->d_column_perm, &v);
    if (st != MIMO_OK || n == 0) return st;
    // the tables are optional; like the permutation they hold batch-global int32 indices
    for (const void *t : {static_cast<const void *>(out->d_positions), static_cast<const void *>(out->d_window_index)}) {
        if (!t) continue;
        if (!aligned16(t)) return MIMO_EALIGN;
        if (v.total_rows > INT32_MAX) return MIMO_EOVERFLOW;
    }
    Tables tables;
    tables.order = out->row_order;
    tables.pos = out->d_positions;
    tables.win = out->d_window_index;
    return launch_range(p, v, 0, n, d_src, src_bytes, src_offsets, heights, widths, channels, out->out_dtype,
                        out->d_out, out->d_column_perm, stream, tables);
}

int mimo_preprocess_units(const mimo_params *p, int32_t n, const uint8_t *d_src, size_t src_bytes,
                          const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                          const int32_t *channels, int64_t first_unit, int64_t unit_count, const mimo_outputs *out,
                          void *stream) {
    if (!out) return MIMO_EINVAL;
    if (out->row_order == MIMO_ORDER_COLUMN) return MIMO_EUNSUPPORTED;
    if (out->row_order != MIMO_ORDER_MERGE) return MIMO_EINVAL;
    if (first_unit < 0 || unit_count < 0) return MIMO_EINVAL;
    Validated v;
    // rows are checked against the window below, not against the whole batch
    int st = validate_batch(p, n, d_src, src_bytes, src_offsets, heights, widths, channels, out->out_dtype,
                            out->d_out, std::numeric_limits<int64_t>::max(), out->d_column_perm, &v);
    if (st != MIMO_OK) return st;
    const int64_t total_units = v.total_rows / 4;
    if (unit_count > total_units || first_unit > total_units - unit_count) return MIMO_ERANGE;
    if (unit_count == 0) return MIMO_OK;
    if (4 * unit_count > out->out_rows_capacity) return MIMO_ECAPACITY;
    for (const void *t : {static_cast<const void *>(out->d_positions), static_cast<const void *>(out->d_window_index)}) {
        if (!t) continue;
        if (!aligned16(t)) return MIMO_EALIGN;
        if (v.total_rows > INT32_MAX) return MIMO_EOVERFLOW;
    }
    Tables tables;
    tables.order = MIMO_ORDER_MERGE;
    tables.pos = out->d_positions;
    tables.win = out->d_window_index;
    UnitWindow win;
    win.lo = first_unit;
    win.hi = first_unit + unit_count;
    win.row_shift = 4 * first_unit;  // rows and positions of the window start at d_out / d_positions
    return launch_range(p, v, 0, n, d_src, src_bytes, src_offsets, heights, widths, channels, out->out_dtype,
                        out->d_out, out->d_column_perm, stream, tables, 0, win);
}

int mimo_preprocess_batch(const mimo_params *p, int32_t n, const uint8_t *d_src, size_t src_bytes,
                          const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                          const int32_t *channels, int32_t out_dtype, void *d_out, int64_t out_rows_capacity,
                          int32_t *d_column_perm, void *stream) {
    mimo_outputs out{};
    out.out_dtype = out_dtype;
    out.row_order = MIMO_ORDER_MERGE;
    out.d_out = d_out;
    out.out_rows_capacity = out_rows_capacity;
    out.d_column_perm = d_column_perm;
    return mimo_preprocess_batch_ex(p, n, d_src, src_bytes, src_offsets, heights, widths, channels, &out, stream);
}

int mimo_preprocess_batch_host(const mimo_params *p, int32_t n, const uint8_t *h_src, size_t src_bytes,
                               const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                               const int32_t *channels, int32_t out_dtype, void *h_out, int64_t out_rows_capacity,
                               int32_t *h_column_perm, uint8_t *d_src_stage, size_t d_src_stage_bytes,
                               void *d_out_stage, int64_t d_out_stage_rows, int32_t *d_perm_stage, void *stream) {
    Validated v;
    int st = validate_batch(p, n, h_src, src_bytes, src_offsets, heights, widths, channels, out_dtype, h_out,
                            out_rows_capacity, h_column_perm, &v);
    if (st != MIMO_OK || n == 0) return st;
    if (!d_src_stage || !d_out_stage) return MIMO_EINVAL;
    if (!aligned16(d_src_stage) || !aligned16(d_out_stage)) return MIMO_EALIGN;
    if (d_src_stage_bytes < src_bytes || d_out_stage_rows < v.total_rows) return MIMO_ECAPACITY;
    if (h_column_perm && (!d_perm_stage || !aligned16(d_perm_stage))) return d_perm_stage ? MIMO_EALIGN : MIMO_EINVAL;

    const size_t row_bytes = static_cast<size_t>(mimo::kRowWidth) * dtype_bytes(out_dtype);
    cudaStream_t caller = static_cast<cudaStream_t>(stream);

    // Chunks of whole images; each chunk's upload -> kernel -> download runs
    // in order on one of two streams, so one chunk's download overlaps the
    // next chunk's upload and kernel. The first chunk holds about 1/64 of the
    // rows and each later one 3x the one before, up to 1/8: the download link
    // then starts after a small upload instead of an eighth of the batch, and
    // each download (3 to 8 bytes out per byte in) still outlasts the next
    // chunk's upload.
    const int64_t target_chunks = std::min<int64_t>(n, 8);
    const int64_t rows_per_chunk = std::max<int64_t>(1, (v.total_rows + target_chunks - 1) / target_chunks);
    int64_t want = std::max<int64_t>(1, rows_per_chunk / 8);

    cudaStream_t ss[2] = {nullptr, nullptr};
    cudaEvent_t start = nullptr;
    int result = MIMO_OK;
    auto fail = [&](cudaError_t e) {
        if (e != cudaSuccess && result == MIMO_OK) result = MIMO_ECUDA;
        return e != cudaSuccess;
    };
    if (fail(cudaStreamCreateWithFlags(&ss[0], cudaStreamNonBlocking)) ||
        fail(cudaStreamCreateWithFlags(&ss[1], cudaStreamNonBlocking)) ||
        fail(cudaEventCreateWithFlags(&start, cudaEventDisableTiming)) || fail(cudaEventRecord(start, caller)) ||
        fail(cudaStreamWaitEvent(ss[0], start, 0)) || fail(cudaStreamWaitEvent(ss[1], start, 0))) {
        // fall through to cleanup
    } else {
        int32_t i = 0;
        int chunk = 0;
        while (i < n && result == MIMO_OK) {
            const int32_t first = i;
            int64_t rows = 0;
            uint64_t lo = UINT64_MAX, hi = 0;
            while (i < n && (rows == 0 || rows + v.plan.img[i].rows <= want)) {
                rows += v.plan.img[i].rows;
                const uint64_t off = static_cast<uint64_t>(src_offsets[i]);
                lo = std::min(lo, off);
                hi = std::max(hi, off + static_cast<uint64_t>(heights[i]) * widths[i] * channels[i]);
                ++i;
            }
            want = std::min(rows_per_chunk, want * 3);
            cudaStream_t s = ss[chunk & 1];
            const int64_t r0 = v.plan.row0[first];
            {
                NvtxRange range("mimo upload");
                if (fail(cudaMemcpyAsync(d_src_stage + lo, h_src + lo, hi - lo, cudaMemcpyHostToDevice, s))) break;
            }
            const int lst = launch_range(p, v, first, i, d_src_stage, src_bytes, src_offsets, heights, widths, channels,
                                         out_dtype, d_out_stage, h_column_perm ? d_perm_stage : nullptr, s);
            if (lst != MIMO_OK) {
                result = lst;
                break;
            }
            NvtxRange download("mimo download");
            if (fail(cudaMemcpyAsync(static_cast<char *>(h_out) + static_cast<size_t>(r0) * row_bytes,
                                     static_cast<char *>(d_out_stage) + static_cast<size_t>(r0) * row_bytes,
                                     static_cast<size_t>(rows) * row_bytes, cudaMemcpyDeviceToHost, s)))
                break;
            if (h_column_perm &&
                fail(cudaMemcpyAsync(h_column_perm + r0, d_perm_stage + r0, sizeof(int32_t) * rows,
                                     cudaMemcpyDeviceToHost, s)))
                break;
            ++chunk;
        }
    }
    NvtxRange wait("mimo wait");
    for (cudaStream_t s : ss) {
        if (s) {
            fail(cudaStreamSynchronize(s));
            cudaStreamDestroy(s);
        }
    }
    if (start) cudaEventDestroy(start);
    return result;
}

int mimo_preprocess_batch_host_noalloc(const mimo_params *p, int32_t n, const uint8_t *h_src, size_t src_bytes,
                                       const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                                       const int32_t *channels, int32_t out_dtype, void *h_out,
                                       int64_t out_rows_capacity, int32_t *h_column_perm, void *stream) {
    Validated v;
    const int st = validate_batch(p, n, h_src, src_bytes, src_offsets, heights, widths, channels, out_dtype, h_out,
                                  out_rows_capacity, h_column_perm, &v);
    if (st != MIMO_OK || n == 0) return st;

    const size_t row_bytes = static_cast<size_t>(mimo::kRowWidth) * dtype_bytes(out_dtype);
    const bool perm = h_column_perm != nullptr;
    auto up = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
    // staged footprint of one image: its bytes (16-byte slots), rows, permutation entries
    auto image_src = [&](int32_t i) {
        return up(static_cast<size_t>(heights[i]) * widths[i] * channels[i], 16);
    };
    auto image_out = [&](int32_t i) {
        const size_t rows = static_cast<size_t>(v.plan.img[i].rows);
        return up(rows * row_bytes, 256) + (perm ? up(rows * sizeof(int32_t), 256) : 0);
    };
    const size_t cap = MIMO_NOALLOC_STAGING_BYTES;
    for (int32_t i = 0; i < n; ++i)
        if (up(image_src(i), 256) + image_out(i) > cap) return MIMO_ELIMIT;

    void *stage = nullptr;
    size_t stage_bytes = 0;
    int rc = mimo::noalloc_staging(&stage, &stage_bytes);
    if (rc != MIMO_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uintptr_t base = reinterpret_cast<uintptr_t>(stage);
    // an error after the first enqueue still waits for what was queued, so
    // that no copy touches the caller's host buffers after the return
    auto bail = [s](int status) {
        cudaStreamSynchronize(s);
        return status;
    };

    // the launch helper reads source offsets by batch index: chunk-local
    // positions go into a batch-sized table
    std::vector<int64_t> local_off(static_cast<size_t>(n), 0);
    int32_t i = 0;
    while (i < n) {
        const int32_t first = i;
        size_t src_used = 0, out_used = 0;
        while (i < n) {
            const size_t s_add = image_src(i), o_add = image_out(i);
            if (i > first && up(src_used + s_add, 256) + out_used + o_add > stage_bytes) break;
            local_off[i] = static_cast<int64_t>(src_used);
            src_used += s_add;
            out_used += o_add;
            ++i;
        }
        const int64_t row0 = v.plan.row0[first];
        const int64_t rows = v.plan.row0[i] - row0;
        const uintptr_t out_at = base + up(src_used, 256);
        const uintptr_t perm_at = out_at + up(static_cast<size_t>(rows) * row_bytes, 256);
        for (int32_t k = first; k < i; ++k) {
            const size_t bytes = static_cast<size_t>(heights[k]) * widths[k] * channels[k];
            if (cudaMemcpyAsync(reinterpret_cast<void *>(base + static_cast<uintptr_t>(local_off[k])),
                                h_src + src_offsets[k], bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return bail(MIMO_ECUDA);
        }
        // The kernel addresses rows and permutation entries by batch-global
        // row index; shifting the bases down by the chunk's first row puts
        // this chunk's rows at the start of its staging slots.
        void *out_base = reinterpret_cast<void *>(out_at - static_cast<uintptr_t>(row0) * row_bytes);
        int32_t *perm_base =
            perm ? reinterpret_cast<int32_t *>(perm_at - static_cast<uintptr_t>(row0) * sizeof(int32_t)) : nullptr;
        rc = launch_range(p, v, first, i, reinterpret_cast<const uint8_t *>(base), src_used, local_off.data(),
                          heights, widths, channels, out_dtype, out_base, perm_base, s);
        if (rc != MIMO_OK) return bail(rc);
        if (cudaMemcpyAsync(static_cast<char *>(h_out) + static_cast<size_t>(row0) * row_bytes,
                            reinterpret_cast<void *>(out_at), static_cast<size_t>(rows) * row_bytes,
                            cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return bail(MIMO_ECUDA);
        if (perm && cudaMemcpyAsync(h_column_perm + row0, reinterpret_cast<void *>(perm_at),
                                    static_cast<size_t>(rows) * sizeof(int32_t), cudaMemcpyDeviceToHost,
                                    s) != cudaSuccess)
            return bail(MIMO_ECUDA);
    }
    return cudaStreamSynchronize(s) == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

int mimo_expand_prompt_ids(const int32_t *ids, int64_t n_ids, int32_t pad_id, const int64_t *counts,
                           int64_t n_items, int32_t *out, int64_t out_capacity, int64_t *out_len) {
    if (n_ids < 0 || n_items < 0 || out_capacity < 0 || !out_len) return MIMO_EINVAL;
    if ((n_ids > 0 && !ids) || (n_items > 0 && !counts) || (out_capacity > 0 && !out)) return MIMO_EINVAL;
    // sizes first: placeholders must match the items one to one
    int64_t pads = 0, total = 0;
    for (int64_t i = 0; i < n_ids; ++i) pads += ids[i] == pad_id;
    if (pads != n_items) return MIMO_EINVAL;
    for (int64_t k = 0; k < n_items; ++k) {
        if (counts[k] < 0 || counts[k] > std::numeric_limits<int64_t>::max() / 2 - total) return MIMO_EINVAL;
        total += counts[k];
    }
    const int64_t len = n_ids - n_items + total;
    if (len > out_capacity) return MIMO_ECAPACITY;
    int64_t k = 0, o = 0;
    for (int64_t i = 0; i < n_ids; ++i) {
        if (ids[i] == pad_id) {
            std::fill(out + o, out + o + counts[k], pad_id);
            o += counts[k++];
        } else {
            out[o++] = ids[i];
        }
    }
    *out_len = len;
    return MIMO_OK;
}

int mimo_patch_embed(const void *d_rows, int64_t rows, const void *d_weight, int32_t embed_dim, const float *d_bias,
                     int32_t out_dtype, void *d_out, int32_t *d_error, void *stream) {
    if (rows < 0 || embed_dim <= 0 || (embed_dim % 256) != 0) return MIMO_EINVAL;
    if (out_dtype != MIMO_F32 && out_dtype != MIMO_BF16) return MIMO_EINVAL;
    if (rows == 0) return MIMO_OK;
    if (!d_rows || !d_weight || !d_out || !d_error) return MIMO_EINVAL;
    if (!aligned16(d_rows) || !aligned16(d_weight) || !aligned16(d_out) || (d_bias && !aligned16(d_bias)) ||
        (reinterpret_cast<uintptr_t>(d_error) & 3u) != 0)
        return MIMO_EALIGN;
    if (rows > (int64_t(1) << 31) - 1) return MIMO_EOVERFLOW;  // TMA coordinates are int32
    return mimo::launch_patch_embed(d_rows, rows, mimo::kRowWidth, d_weight, embed_dim, d_bias, out_dtype, d_out,
                                    d_error, stream);
}

int mimo_patch_embed_stall_test(const void *d_rows, int64_t rows, const void *d_weight, int32_t embed_dim,
                                const float *d_bias, int32_t out_dtype, void *d_out, int32_t *d_error,
                                int32_t stop_after_kblocks, uint32_t wait_rounds, void *stream) {
    if (rows <= 0 || embed_dim <= 0 || (embed_dim % 256) != 0) return MIMO_EINVAL;
    if (out_dtype != MIMO_F32 && out_dtype != MIMO_BF16) return MIMO_EINVAL;
    if (stop_after_kblocks < 0 || stop_after_kblocks > mimo::kRowWidth / 128 || wait_rounds == 0) return MIMO_EINVAL;
    if (!d_rows || !d_weight || !d_out || !d_error) return MIMO_EINVAL;
    if (!aligned16(d_rows) || !aligned16(d_weight) || !aligned16(d_out) || (d_bias && !aligned16(d_bias)) ||
        (reinterpret_cast<uintptr_t>(d_error) & 3u) != 0)
        return MIMO_EALIGN;
    if (rows > (int64_t(1) << 31) - 1) return MIMO_EOVERFLOW;
    return mimo::launch_patch_embed(d_rows, rows, mimo::kRowWidth, d_weight, embed_dim, d_bias, out_dtype, d_out,
                                    d_error, stream, wait_rounds, stop_after_kblocks);
}

int mimo_preprocess_embed(const mimo_params *p, int32_t n, const uint8_t *d_src, size_t src_bytes,
                          const int64_t *src_offsets, const int32_t *heights, const int32_t *widths,
                          const int32_t *channels, int32_t row_order, const void *d_weight, int32_t embed_dim,
                          const float *d_bias, int32_t out_dtype, void *d_out, int64_t out_rows_capacity,
                          void *d_scratch, size_t scratch_bytes, int32_t *d_error, void *stream) {
    if (row_order != MIMO_ORDER_MERGE && row_order != MIMO_ORDER_COLUMN) return MIMO_EINVAL;
    if (embed_dim <= 0 || (embed_dim % 256) != 0) return MIMO_EINVAL;
    Validated v;
    int st = validate_batch(p, n, d_src, src_bytes, src_offsets, heights, widths, channels, out_dtype, d_out,
                            out_rows_capacity, nullptr, &v);
    if (st != MIMO_OK || n == 0) return st;
    if (!d_weight || !d_scratch || !d_error) return MIMO_EINVAL;
    if (!aligned16(d_weight) || !aligned16(d_scratch) || (d_bias && !aligned16(d_bias)) ||
        (reinterpret_cast<uintptr_t>(d_error) & 3u) != 0)
        return MIMO_EALIGN;
    if (v.total_rows > (int64_t(1) << 31) - 1) return MIMO_EOVERFLOW;
    // runs of whole images alternate between the two halves of the scratch. The pixel kernel of run r
    // goes on the caller's stream, the GEMM of run r on a stream of the library's that belongs to its
    // half, so that it overlaps the pixel kernel of run r + 1 (the unstaged pixel kernel holds no shared
    // memory and fits beside the GEMM's CTAs) and the GEMM of run r + 1 can start on the SMs that the
    // last, partial wave of run r's tiles leaves idle. Events order each GEMM after its run's rows and
    // each reuse of a half after the GEMM that read it; the caller's stream finally waits for both.
    // (Four slots of one run each, rotating, measured no faster than two halves.)
    const int64_t row_bytes = static_cast<int64_t>(mimo::kRowWidth) * 2;
    const int64_t run_rows = static_cast<int64_t>(scratch_bytes / 2) / row_bytes;
    for (int32_t i = 0; i < n; ++i)
        if (v.plan.row0[i + 1] - v.plan.row0[i] > run_rows) return MIMO_ECAPACITY;  // exceeds half the scratch
    // the two streams and their events, made once per host thread and device
    struct Aux {
        bool ready = false;
        cudaStream_t s[2] = {nullptr, nullptr};
        cudaEvent_t rows_ready[2] = {nullptr, nullptr}, rows_read[2] = {nullptr, nullptr};
    };
    constexpr int kMaxDevices = 64;
    static thread_local Aux aux_of[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MIMO_ECUDA;
    Aux &aux = aux_of[dev];
    if (!aux.ready) {
        // handles made before a failed creation are kept and reused by the next attempt
        for (int k = 0; k < 2; ++k)
            if ((!aux.s[k] && cudaStreamCreateWithFlags(&aux.s[k], cudaStreamNonBlocking) != cudaSuccess) ||
                (!aux.rows_ready[k] && cudaEventCreateWithFlags(&aux.rows_ready[k], cudaEventDisableTiming) !=
                                           cudaSuccess) ||
                (!aux.rows_read[k] &&
                 cudaEventCreateWithFlags(&aux.rows_read[k], cudaEventDisableTiming) != cudaSuccess))
                return MIMO_ECUDA;
        aux.ready = true;
    }
    cudaStream_t main_s = static_cast<cudaStream_t>(stream);
    // an error after the first enqueue waits for the library streams' work, so
    // that no GEMM still reads the scratch or writes d_out after the return
    auto bail = [&aux](int status) {
        cudaStreamSynchronize(aux.s[0]);
        cudaStreamSynchronize(aux.s[1]);
        return status;
    };
    uint8_t *halves[2] = {static_cast<uint8_t *>(d_scratch), static_cast<uint8_t *>(d_scratch) + run_rows * row_bytes};
    const size_t esz = out_dtype == MIMO_BF16 ? 2 : 4;
    Tables tables;
    tables.order = row_order;
    int run = 0;
    for (int32_t i0 = 0; i0 < n; ++run) {
        int32_t i1 = i0;
        while (i1 < n && v.plan.row0[i1 + 1] - v.plan.row0[i0] <= run_rows) ++i1;
        if (i1 == i0) return bail(MIMO_ECAPACITY);  // one image's rows exceed half the scratch
        const int h = run & 1;
        const int64_t row_base = v.plan.row0[i0];
        const int64_t rows = v.plan.row0[i1] - row_base;
        if (run >= 2 && cudaStreamWaitEvent(main_s, aux.rows_read[h], 0) != cudaSuccess) return bail(MIMO_ECUDA);
        st = launch_range(p, v, i0, i1, d_src, src_bytes, src_offsets, heights, widths, channels, MIMO_BF16,
                          halves[h], nullptr, stream, tables, row_base, UnitWindow(), true);
        if (st != MIMO_OK) return bail(st);
        if (cudaEventRecord(aux.rows_ready[h], main_s) != cudaSuccess ||
            cudaStreamWaitEvent(aux.s[h], aux.rows_ready[h], 0) != cudaSuccess)
            return bail(MIMO_ECUDA);
        st = mimo::launch_patch_embed(halves[h], rows, mimo::kRowWidth, d_weight, embed_dim, d_bias, out_dtype,
                                      static_cast<uint8_t *>(d_out) + static_cast<size_t>(row_base) * embed_dim * esz,
                                      d_error, aux.s[h]);
        if (st != MIMO_OK) return bail(st);
        // the half has been read: drop its rows from L2 without writing them back to HBM (a scratch that
        // is not 128-byte aligned keeps them; they are then written back as usual)
        st = mimo::launch_discard_l2(halves[h], rows * row_bytes, aux.s[h]);
        if (st != MIMO_OK && st != MIMO_EALIGN) return bail(st);
        if (cudaEventRecord(aux.rows_read[h], aux.s[h]) != cudaSuccess) return bail(MIMO_ECUDA);
        i0 = i1;
    }
    // the caller's stream sees every GEMM done
    for (int h = 0; h < 2 && h < run; ++h)
        if (cudaStreamWaitEvent(main_s, aux.rows_read[h], 0) != cudaSuccess) return bail(MIMO_ECUDA);
    return MIMO_OK;
}

const char *mimo_status_string(int status) {
    switch (status) {
        case MIMO_OK: return "ok";
        case MIMO_EINVAL: return "invalid argument";
        case MIMO_EASPECT: return "absolute aspect ratio must be at most 200";
        case MIMO_EDEGENERATE: return "max_pixels shrink rounds a side down to zero";
        case MIMO_ECHANNELS: return "channels must be 3 (RGB) or 4 (RGBA)";
        case MIMO_EUNSUPPORTED: return "unsupported processor knobs (patch 16, temporal 2, merge 2, std > 0)";
        case MIMO_EALIGN: return "source offsets and output pointers must be 16-byte aligned";
        case MIMO_ECAPACITY: return "output or staging buffer too small for the batch";
        case MIMO_EOVERFLOW: return "size exceeds the supported index range";
        case MIMO_ECUDA: return "CUDA runtime error";
        case MIMO_ERANGE: return "an image lies outside the source buffer";
        case MIMO_ELIMIT: return "an image does not fit the fixed staging area of the no-allocation entry point";
        default: return "unknown status";
    }
}

int mimo_bounds_check_status(int64_t *violations, int32_t *first_kind) {
    if (!violations || !first_kind) return MIMO_EINVAL;
    return mimo::bounds_check_status(violations, first_kind);
}

int mimo_version(void) { return 10000; }

}  // extern "C"

// ---------------------------------------------------------------- video
namespace {

int64_t video_budget(int64_t n, int64_t total_max, const mimo_params *p) {
    if (total_max <= 0) return p->max_pixels;
    const int64_t share = (total_max * p->temporal_patch_size) / n;
    return std::max<int64_t>(p->min_pixels, std::min<int64_t>(share, p->max_pixels));
}

struct VideoPlan {
    ImagePlan ip;
    int64_t gt = 0, rows = 0;
};

int plan_video(int32_t n_frames, int32_t height, int32_t width, int64_t total_max, const mimo_params *p,
               VideoPlan *vp) {
    int st = check_params(p);
    if (st != MIMO_OK) return st;
    if (n_frames <= 0 || height <= 0 || width <= 0) return MIMO_EINVAL;
    if (total_max > std::numeric_limits<int64_t>::max() / 4) return MIMO_EOVERFLOW;
    mimo_params q = *p;
    q.max_pixels = video_budget(n_frames, total_max, p);
    st = plan_image(height, width, &q, &vp->ip);
    if (st != MIMO_OK) return st;
    vp->gt = (static_cast<int64_t>(n_frames) + 1) / 2;  // an odd count repeats its last frame
    if (vp->ip.blocks * vp->gt * 2 > INT32_MAX) return MIMO_EOVERFLOW;
    vp->rows = vp->gt * vp->ip.rows;
    return MIMO_OK;
}

}  // namespace

extern "C" {

int mimo_video_max_pixels(int64_t n_sampled, int64_t total_max_pixels, const mimo_params *p, int64_t *out) {
    if (!p || !out || n_sampled <= 0 || total_max_pixels < 0) return MIMO_EINVAL;
    if (total_max_pixels > std::numeric_limits<int64_t>::max() / 4) return MIMO_EOVERFLOW;
    *out = video_budget(n_sampled, total_max_pixels, p);
    return MIMO_OK;
}

int mimo_smart_nframes(int64_t total, double fps_src, double fps, int64_t min_frames, int64_t max_frames,
                       int64_t *out) {
    if (!out || total <= 0 || !(fps_src > 0.0) || !(fps > 0.0) || min_frames < 0 || max_frames < min_frames)
        return MIMO_EINVAL;
    const double n = std::min(std::min(std::max(static_cast<double>(total) / fps_src * fps,
                                                static_cast<double>(min_frames)),
                                       static_cast<double>(max_frames)),
                              static_cast<double>(total));
    const int64_t even = 2 * static_cast<int64_t>(std::floor(n * 0.5));
    if (even <= 0) return MIMO_EINVAL;
    *out = even;
    return MIMO_OK;
}

int mimo_sample_frames(int64_t total, int64_t n, double fps_src, int64_t *idx, float *ts, int64_t *count) {
    if (total <= 0 || n <= 0 || !(fps_src > 0.0) || !idx || !ts || !count) return MIMO_EINVAL;
    const double last = static_cast<double>(total - 1);
    const double step = n > 1 ? last / static_cast<double>(n - 1) : 0.0;
    const float rate = static_cast<float>(fps_src);
    int64_t k = 0;
    for (int64_t j = 0; j < n; ++j) {
        const int64_t i = (n > 1 && j == n - 1) ? total - 1 : static_cast<int64_t>(static_cast<double>(j) * step);
        if (k == 0 || idx[k - 1] != i) {
            idx[k] = i;
            ts[k] = static_cast<float>(i) / rate;
            ++k;
        }
    }
    *count = k;
    return MIMO_OK;
}

int mimo_plan_video(int32_t n_frames, int32_t height, int32_t width, int64_t total_max_pixels,
                    const mimo_params *p, int64_t *grid_thw, int64_t *rows) {
    if (!grid_thw || !rows) return MIMO_EINVAL;
    VideoPlan vp;
    const int st = plan_video(n_frames, height, width, total_max_pixels, p, &vp);
    if (st != MIMO_OK) return st;
    grid_thw[0] = vp.gt;
    grid_thw[1] = vp.ip.Hr / 16;
    grid_thw[2] = vp.ip.Wr / 16;
    *rows = vp.rows;
    return MIMO_OK;
}

int mimo_preprocess_video(const mimo_params *p, int32_t n_frames, const uint8_t *d_frames, size_t src_bytes,
                          int64_t frame_stride, int32_t height, int32_t width, int32_t channels,
                          int64_t total_max_pixels, const mimo_outputs *out, void *stream) {
    if (!out || !d_frames) return MIMO_EINVAL;
    if (out->row_order != MIMO_ORDER_MERGE && out->row_order != MIMO_ORDER_COLUMN) return MIMO_EINVAL;
    if (out->out_dtype != MIMO_F32 && out->out_dtype != MIMO_BF16) return MIMO_EINVAL;
    if (channels != 3 && channels != 4) return MIMO_ECHANNELS;
    VideoPlan vp;
    int st = plan_video(n_frames, height, width, total_max_pixels, p, &vp);
    if (st != MIMO_OK) return st;
    const uint64_t frame_bytes = static_cast<uint64_t>(height) * static_cast<uint64_t>(width) * channels;
    if (frame_stride < 0 || static_cast<uint64_t>(frame_stride) < frame_bytes) return MIMO_EINVAL;
    if ((frame_stride & 15) != 0 || !aligned16(d_frames) || !aligned16(out->d_out)) return MIMO_EALIGN;
    const uint64_t need = static_cast<uint64_t>(n_frames - 1) * static_cast<uint64_t>(frame_stride) + frame_bytes;
    if (need > src_bytes) return MIMO_ERANGE;
    if (vp.rows > out->out_rows_capacity) return MIMO_ECAPACITY;
    if (!out->d_out) return MIMO_EINVAL;
    for (const void *t : {static_cast<const void *>(out->d_column_perm), static_cast<const void *>(out->d_positions),
                          static_cast<const void *>(out->d_window_index)}) {
        if (!t) continue;
        if (!aligned16(t)) return MIMO_EALIGN;
        if (vp.rows > INT32_MAX) return MIMO_EOVERFLOW;
    }

    static thread_local mimo::LaunchParams lp;
    std::memset(&lp, 0, sizeof(lp));
    lp.src = d_frames;
    lp.out = out->d_out;
    lp.perm = out->d_column_perm;
    lp.pos = out->d_positions;
    lp.win = out->d_window_index;
    lp.order = out->row_order;
    fold_normalisation(p, &lp);
    mimo::ImageDesc &d = lp.img[0];
    d.src_off = 0;
    d.row0 = 0;
    d.limit = static_cast<int64_t>(src_bytes);
    d.frame_stride = frame_stride;
    d.H = height;
    d.W = width;
    d.Hr = static_cast<int32_t>(vp.ip.Hr);
    d.Wr = static_cast<int32_t>(vp.ip.Wr);
    d.flags = vp.ip.flags | mimo::kVideo | (channels << mimo::kChannelShift);
    d.frames = n_frames;
    const int64_t blocks = vp.ip.blocks * vp.gt * 2;  // (t, block, tt) halves
    lp.block_start[0] = 0;
    lp.block_start[1] = static_cast<int32_t>(blocks);
    lp.n = 1;
    lp.tile_rows = vp.ip.tile_rows;
    lp.tile_stride = (std::max(vp.ip.tile_cols, mimo::kBlock) + 3) & ~3;
    const size_t tile_floats = 3u * static_cast<size_t>(lp.tile_rows) * static_cast<size_t>(lp.tile_stride);
    lp.raw_stride = ((32 + 4 * vp.ip.tile_cols) + 15) & ~15;
    const size_t raw_floats = static_cast<size_t>(lp.tile_rows) * static_cast<size_t>(lp.raw_stride) / 4u;
    lp.raw = static_cast<int32_t>(tile_floats);
#if defined(MIMO_BOUNDS_CHECK)
    lp.chk_row_lo = 0;
    lp.chk_row_hi = vp.rows;
    lp.chk_table_rows = vp.rows;
    lp.chk_smem_floats = static_cast<int32_t>(tile_floats + raw_floats);
#endif
    return mimo::launch_preprocess(lp, blocks, out->out_dtype, sizeof(float) * (tile_floats + raw_floats), stream);
}

}  // extern "C"
