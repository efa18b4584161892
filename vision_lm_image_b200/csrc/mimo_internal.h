// mimo_internal.h -- types shared by the host planner (mimo_api.cpp) and the
// sm_100a kernel (mimo_preprocess.cu). Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#if defined(__CUDACC__)
#define MIMO_HD __host__ __device__ __forceinline__
#else
#define MIMO_HD inline
#endif

namespace mimo {

// One 32x32 output merge block at a time per CTA; the source samples it
// needs are staged in shared memory as planar fp32 tiles of at most kMaxTile
// rows and columns (2 taps x 32 outputs).
constexpr int kBlock = 32;             // merge block side in resized pixels (patch 16 x merge 2)
constexpr int kRowWidth = 1536;        // 3 channels x 2 frames x 16 x 16
constexpr int kMaxTile = 64;           // 32 outputs x 2 taps
constexpr int kThreads = 256;
constexpr int kMaxImagesPerLaunch = 512;

// Per-axis staging mode of an image, decided on the host:
//  - gathered: the block's source span does not fit kMaxTile, so only the
//    two taps of each of the 32 outputs are staged (tile index 2d, 2d+1);
//  - identity: the axis is not resized (in == out), every weight is 0 and
//    only the first tap of each output is staged (32 entries);
//  - otherwise the span from the first to the last tap is staged whole.
enum : int32_t { kGatherRows = 1, kGatherCols = 2, kIdentityRows = 4, kIdentityCols = 8, kVideo = 16 };
constexpr int kChannelShift = 8;  // channels (3 or 4) live in bits 8..15 of the flags

// One image, or one video whose consecutive frames pair up as temporal
// patches. A video's blocks are (t, block row, block col, tt) halves, tt
// innermost: each half stages frame min(2t + tt, frames - 1) and writes the
// temporal slot tt of its merge unit's rows.
struct ImageDesc {
    int64_t src_off;       // byte offset of the (first) frame in the source buffer
    int64_t row0;          // first output row of the item in the batch
    int64_t limit;         // bytes of the caller's source buffer from src_off on
    int64_t frame_stride;  // bytes from one frame to the next (videos)
    int32_t H, W;          // source size
    int32_t Hr, Wr;        // resized size, multiples of 32
    int32_t flags;         // kGather* | kIdentity* | kVideo | channels << kChannelShift
    int32_t frames;        // source frames (1 for an image)
};
static_assert(sizeof(ImageDesc) == 56, "descriptor layout");

// Debug builds compiled with -DMIMO_BOUNDS_CHECK check every global load and
// store of the pixel kernels (and their shared-memory tile indices) against the
// extents they must stay in: the image's bytes and the caller's source buffer,
// the output rows and tables the host validated. A failed check skips the
// access and counts it in a device status word (mimo_bounds_check_status); it
// never traps. Release builds compile the checks away.
#if defined(MIMO_BOUNDS_CHECK)
#define MIMO_CHECK(cond, kind) (::mimo::bounds_ok((cond), (kind)))
#else
#define MIMO_CHECK(cond, kind) true
#endif
enum : int32_t {
    kChkSrcCopy = 1,     // staged source copy outside the caller's buffer
    kChkSrcLoad = 2,     // direct source load outside the image
    kChkSmem = 3,        // shared-memory tile or staging index outside its region
    kChkRowStore = 4,    // output row outside the validated rows
    kChkTableStore = 5,  // permutation / position / window entry outside its table
};

// Everything one launch needs travels by value as the kernel's parameter
// block (__grid_constant__), so a launch needs no device-side table and no
// host-to-device copy. The block is sized for kCap images: the driver copies
// all of it on every launch, so launches of a few images use a small one.
template <int kCap>
struct LaunchParamsT {
    const uint8_t *src;
    void *out;
    int32_t *perm;       // may be null
    int32_t *pos;        // may be null: (patch row, patch column) per emitted row
    int32_t *win;        // may be null: merge-order unit of each column-major unit
    int32_t order;       // 0: merge-block order, 1: column order
    int32_t unit0;       // first merge unit of img[0] in this launch (a launch may start inside an image)
    float k[3], b[3];    // normalisation folded: v = x*k[c] + b[c]
    int32_t n;           // images in this launch
    int32_t tile_rows;   // rows of the shared-memory tile (max over images)
    int32_t tile_stride; // row stride (floats, multiple of 4) of the tile
    int32_t raw;         // float offset of the raw staging rows
    int32_t raw_stride;  // bytes per raw staging row (multiple of 16)
    int32_t keep_rows;   // bf16 rows read again right away (chained patch embedding): stored with L2 evict-last
    int32_t warp_rows;   // warp-staged kernel: source rows a warp stages per block (max over images)
    int32_t warp_stride; // warp-staged kernel: bytes per staged row (multiple of 16)
#if defined(MIMO_BOUNDS_CHECK)
    int64_t chk_row_lo, chk_row_hi;  // rows the kernel may emit (its own row numbering)
    int64_t chk_table_rows;          // rows the permutation covers (window index: a quarter)
    int32_t chk_smem_floats;         // floats of dynamic shared memory (tile + raw)
    int32_t chk_pad;
#endif
    int32_t block_start[kCap + 1];  // prefix sum of blocks (video blocks are halves)
    ImageDesc img[kCap];
};
using LaunchParams = LaunchParamsT<kMaxImagesPerLaunch>;
constexpr int kSmallLaunch = 32;  // launches of up to this many images use the small block
using SmallLaunchParams = LaunchParamsT<kSmallLaunch>;
static_assert(sizeof(LaunchParams) <= 32764 - 64, "kernel parameter limit");

// Bilinear taps of output index d along an axis of size in -> out under the
// align_corners=False rule, computed exactly: the source coordinate is the
// rational ((2d+1)*in - out) / (2*out), clamped at 0 from below.
struct Taps {
    int64_t i0, i1;
    int64_t rem, den;  // weight of the second tap = rem / den
};

MIMO_HD Taps axis_taps(int64_t d, int64_t in, int64_t out) {
    Taps t;
    const int64_t num = (2 * d + 1) * in - out;
    t.den = 2 * out;
    if (num <= 0) {
        t.i0 = 0;
        t.rem = 0;
    } else {
        t.i0 = num / t.den;
        t.rem = num - t.i0 * t.den;
    }
    t.i1 = (t.i0 + 1 < in) ? t.i0 + 1 : in - 1;
    return t;
}

// Number of source rows (or columns) a merge block touches when staged
// contiguously: last tap of output 32b+31 minus first tap of output 32b, + 1.
MIMO_HD int64_t block_span(int64_t b, int64_t in, int64_t out) {
    const Taps first = axis_taps(b * kBlock, in, out);
    const Taps last = axis_taps(b * kBlock + kBlock - 1, in, out);
    return last.i1 - first.i0 + 1;
}

int launch_preprocess(const LaunchParams &lp, int64_t blocks, int out_dtype, size_t smem_bytes, void *stream);

// Drops `bytes` from `p` (128-byte aligned) out of L2 without writing them back
// (their contents become undefined), on `stream`.
int launch_discard_l2(void *p, int64_t bytes, void *stream);

#if defined(MIMO_BOUNDS_CHECK) && defined(__CUDACC__)
__device__ bool bounds_ok(bool ok, int kind);
#endif
// Failed bounds checks since the last query, and the kind of the first
// (MIMO_EUNSUPPORTED unless built with -DMIMO_BOUNDS_CHECK); clears both.
int bounds_check_status(int64_t *violations, int32_t *first_kind);

// Patch embedding GEMM on the tensor cores (mimo_patch_embed.cu). wait_rounds
// = 0 keeps the default wait limit; stop_after >= 0 (tests of the failure path
// only) stops each CTA's operand loaders after that many 128-wide K blocks.
int launch_patch_embed(const void *d_rows, int64_t M, int32_t K, const void *d_weight, int32_t N, const float *d_bias,
                       int32_t out_dtype, void *d_out, int32_t *d_err, void *stream, uint32_t wait_rounds = 0,
                       int32_t stop_after = -1);

// Device address and size of the library's fixed staging area on the
// current device (mimo_noalloc.cu).
int noalloc_staging(void **dev_ptr, size_t *bytes);

}  // namespace mimo
