// mimo_preprocess.cu -- the fused MiMo-V2 pixel path for sm_100a.
//
// The unit of work is one 32x32 merge block of one resized image (4 output
// rows of 1536 values). For each block the kernel
//   - computes the exact bilinear taps of its 32 output rows (warp 0) and 32
//     output columns (warp 1) under align_corners=False (NeMo Automodel
//     "mimo_v2_flash.processing", class MimoV2ImageProcessor: F.interpolate
//     bilinear; docs.rs "cortiq_engine::mimo_vision", resize_bilinear);
//   - copies the source row segments those taps touch into shared memory
//     with 16-byte cp.async, then converts them to planar fp32 on the 0..255
//     scale, compositing RGBA onto white on the way (function _to_rgb);
//   - interpolates along W for every staged row, in place (skipped when the
//     width is not resized; for RGB images this step and the conversion are
//     one: each job reads its output columns' two taps straight from the
//     staged bytes), then along H with packed f32x2 arithmetic, applies
//     (x - 255*mean)/(255*std) folded to x*k + b (module docstring), and
//     writes each 16-pixel row segment twice, once per temporal frame, laid
//     out (c, tt, py, px) in merge-block row order (cortiq page, conventions);
//   - writes the column-order permutation entries of its merge unit (cortiq
//     page, column_permutation).
// CTAs are persistent: each takes a contiguous range of blocks and overlaps
// the source copies of the next blocks with the stores of the current one.
// The staged kernel is instantiated with and without the fused RGB step; a
// launch takes the fused one only when one of its images needs it. Launches
// whose images or frames all keep their width go to a second, unstaged kernel
// (direct_kernel below) when that measured faster, and launches that shrink
// every image's height by 1.25 or more to a third, warp-staged one
// (warp_kernel below).
// There is no inter-CTA communication, no atomics and no global wait; every
// output element has exactly one writer.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstring>

#include "mimo.h"
#include "mimo_internal.h"

namespace mimo {

#if defined(MIMO_BOUNDS_CHECK)
// Debug builds: accesses that failed their bounds check (skipped, not made),
// and the kind of the first one.
__device__ unsigned long long g_bounds_violations;
__device__ int g_bounds_first_kind;

__device__ __noinline__ bool bounds_ok(bool ok, int kind) {
    if (!ok) {
        atomicAdd(&g_bounds_violations, 1ull);
        atomicCAS(&g_bounds_first_kind, 0, kind);
    }
    return ok;
}
#endif

namespace {

constexpr float kTwo23 = 8388608.0f;
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer

// Byte k of w as the float 2^23 + byte: PRMT builds the bit pattern
// 0x4B0000bb; subtracting 2^23 afterwards gives the byte value exactly.
template <int k>
__device__ __forceinline__ float byte_bits(uint32_t w) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u + k));
}
template <int k>
__device__ __forceinline__ float byte_f(uint32_t w) {
    return byte_bits<k>(w) - kTwo23;
}

// Packed fp32 pairs: sm_100 executes one FMA/ADD on both halves of a float2.
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Composite channel pairs onto white: nearest integer of (c*a + 255*(255-a))
// / 255 per lane of the pair. c*a + white is an exact integer below 2^24;
// t/255 is never within 1/510 of a half-integer (255 is odd) while the
// product with fl(1/255) is within 1e-5 of it, so one FMA with the 1.5*2^23
// constant rounds it exactly.
__device__ __forceinline__ float2 on_white2(float2 c2, float2 a2, float2 white2) {
    const float2 t = fma2(c2, a2, white2);
    return add2(fma2(t, f2(1.0f / 255.0f, 1.0f / 255.0f), f2(kRound, kRound)), f2(-kRound, -kRound));
}

// last i with block_start[i] <= blk
template <class Params>
__device__ __forceinline__ int find_image(const Params &P, int blk) {
    int lo = 0, hi = P.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.block_start[mid] <= blk) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Taps, staging geometry and output addresses of one merge block (double-
// buffered in shared memory: the pipeline holds the current block and the
// next one). Every later phase reads the block's constants from here.
struct alignas(16) TapSet {  // 16-byte aligned; the fused RGB path reads tap pairs as int2 / float2
    int32_t ty[2][kBlock];   // tile row of each output row's two taps
    int32_t tx[2][kBlock];   // tile column of each output column's two taps
    float ly[kBlock];        // weight of the second row tap
    float lx[kBlock];        // weight of the second column tap
    int32_t srow[kMaxTile];  // source row of each tile row (gathered rows)
    int32_t scol[kMaxTile];  // source column of each tile column (gathered columns)
    int32_t y_first, nrows;  // first source row / staged rows (contiguous rows)
    int32_t x_first, ncols;  // first source column / staged columns
    int32_t flags, W, C, CQ; // image flags, width, channels, 16-byte chunks per staged row
    int32_t gw2, gh2, bh, bw;
    int32_t t, tt;            // temporal patch and slot (videos; 0 for images)
    int32_t Q, pad_q;          // staging jobs (4 pixels) per tile row
    uint32_t qmagic, cmagic;  // x / Q and x / CQ as (x * magic) >> 16 for the job counts here
    int64_t src_off;         // image offset in the source buffer
    int64_t limit;           // bytes readable from src_off (caller's buffer end)
    int64_t row0;            // first output row of the image
    int64_t row_base;        // first output row of the block, in the emitted order
};

// Per-lane state of a tap warp across the blocks of a CTA: the exact floor
// quotient q and remainder r of ((2d+1)*in - out) / (2*out) for the lane's
// output index d in the last block seen along the warp's axis, and the
// change of both from one block to the next.
struct AxisCursor {
    int blk = -2, ii = 0, t = 0, bh = 0, bw = 0, tt = 0;  // position of the last block handled
    int img = -1, b = -2;
    // q <= in and r < den = 2 * out: both fit 32 bits (only the first numerator needs 64)
    int32_t q = 0, r = 0;
    int32_t den = 1, step_q = 0, step_r = 0;
    double inv_den = 1.0;
    float inv_den_f = 1.0f;
};

// ceil(65536 / n) for n = 1..18 (entry 0 unused): x / n = (x * entry) >> 16
// for the job indices below (x < 64 * n), looked up instead of divided
constexpr uint32_t ceil_65536(uint32_t n) { return (65536u + n - 1) / n; }
__constant__ uint32_t kCeil65536[19] = {0,
                                        ceil_65536(1),  ceil_65536(2),  ceil_65536(3),  ceil_65536(4),
                                        ceil_65536(5),  ceil_65536(6),  ceil_65536(7),  ceil_65536(8),
                                        ceil_65536(9),  ceil_65536(10), ceil_65536(11), ceil_65536(12),
                                        ceil_65536(13), ceil_65536(14), ceil_65536(15), ceil_65536(16),
                                        ceil_65536(17), ceil_65536(18)};

// Warps 0 (rows) and 1 (columns): taps of block blk into T. `prev` holds the
// taps of the block before blk in this CTA's order.
template <class Params>
__device__ __forceinline__ void compute_taps(const Params &P, TapSet &T, const TapSet &prev, int blk,
                                             AxisCursor &cur, int warp, int lane) {
    // block position: consecutive blocks advance one column (or start the
    // next block row / temporal patch / item), a video first through its
    // two temporal halves; only the CTA's first block needs divisions
    int ii = cur.ii, t, bh, bw, tt;
    if (blk == cur.blk + 1) {
        if (ii + 1 < P.n && P.block_start[ii + 1] <= blk) {
            ++ii;
            t = bh = bw = tt = 0;
        } else {
            const ImageDesc &Dc = P.img[ii];
            t = cur.t;
            bh = cur.bh;
            bw = cur.bw;
            tt = cur.tt;
            if ((Dc.flags & kVideo) != 0 && tt == 0) {
                tt = 1;
            } else {
                tt = 0;
                if (++bw == Dc.Wr / kBlock) {
                    bw = 0;
                    if (++bh == Dc.Hr / kBlock) {
                        bh = 0;
                        ++t;
                    }
                }
            }
        }
    } else {
        ii = find_image(P, blk);
        const ImageDesc &Dc = P.img[ii];
        // the launch's first image may start at merge unit unit0 (image launches only)
        int local = blk - P.block_start[ii] + (ii == 0 ? P.unit0 : 0);
        const bool vid = (Dc.flags & kVideo) != 0;
        tt = vid ? (local & 1) : 0;
        if (vid) local >>= 1;
        const int g = Dc.Wr / kBlock;
        const int units = (Dc.Hr / kBlock) * g;
        t = local / units;
        local -= t * units;
        bh = local / g;
        bw = local - bh * g;
    }
    cur.blk = blk;
    cur.ii = ii;
    cur.t = t;
    cur.bh = bh;
    cur.bw = bw;
    cur.tt = tt;
    const ImageDesc &D = P.img[ii];
    const int32_t H = D.H, W = D.W, Hr = D.Hr, Wr = D.Wr, flags = D.flags;
    const int32_t C = (flags >> kChannelShift) & 0xFF;
    const int gw2 = Wr / kBlock;
    const bool is_col = warp == 1;
    const int64_t in = is_col ? W : H;
    const int64_t out = is_col ? Wr : Hr;
    const int b = is_col ? bw : bh;

    if (ii == cur.img && b == cur.b) {
        // same block row (column) as the previous block: its taps are unchanged
        if (!is_col) {
            T.ty[0][lane] = prev.ty[0][lane];
            T.ty[1][lane] = prev.ty[1][lane];
            T.ly[lane] = prev.ly[lane];
            T.srow[lane] = prev.srow[lane];
            T.srow[lane + 32] = prev.srow[lane + 32];
            if (lane == 0) {
                T.y_first = prev.y_first;
                T.nrows = prev.nrows;
            }
        } else {
            T.tx[0][lane] = prev.tx[0][lane];
            T.tx[1][lane] = prev.tx[1][lane];
            T.lx[lane] = prev.lx[lane];
            T.scol[lane] = prev.scol[lane];
            T.scol[lane + 32] = prev.scol[lane + 32];
            if (lane == 0) {
                T.x_first = prev.x_first;
                T.ncols = prev.ncols;
                T.CQ = prev.CQ;
                T.Q = prev.Q;
                T.cmagic = prev.cmagic;
                T.qmagic = prev.qmagic;
            }
        }
    } else {
        if (ii != cur.img) {
            cur.img = ii;
            cur.b = -2;
            cur.den = static_cast<int32_t>(2 * out);
            cur.inv_den = 1.0 / static_cast<double>(cur.den);
            cur.inv_den_f = static_cast<float>(cur.inv_den);
            const int64_t step = 2 * kBlock * in;  // numerator change between blocks
            const int64_t sq = step / cur.den;
            cur.step_q = static_cast<int32_t>(sq);
            cur.step_r = static_cast<int32_t>(step - sq * cur.den);
        }
        if (b == cur.b + 1) {
            cur.q += cur.step_q;
            cur.r += cur.step_r;
            if (cur.r >= cur.den) {
                cur.r -= cur.den;
                ++cur.q;
            }
        } else {
            // floor division of the (possibly negative) numerator: fp64
            // estimate, exact integer correction
            const int64_t d = static_cast<int64_t>(b) * kBlock + lane;
            const int64_t num = (2 * d + 1) * in - out;
            int64_t q = static_cast<int64_t>(floor(static_cast<double>(num) * cur.inv_den));
            int64_t r = num - q * cur.den;
            while (r < 0) {
                --q;
                r += cur.den;
            }
            while (r >= cur.den) {
                ++q;
                r -= cur.den;
            }
            cur.q = static_cast<int32_t>(q);
            cur.r = static_cast<int32_t>(r);
        }
        cur.b = b;
        // source coordinate clamped at 0: negative quotient -> first pixel, weight 0
        const bool clamp = cur.q < 0;
        const int32_t i0 = clamp ? 0 : static_cast<int32_t>(cur.q);
        const int32_t i1 = (static_cast<int64_t>(i0) + 1 < in) ? i0 + 1 : static_cast<int32_t>(in - 1);
        // r < den; below 2^23 the float conversion is exact with the 2^23 bit trick
        const float rf = (cur.r < (1 << 23))
                             ? __uint_as_float(0x4B000000u | static_cast<uint32_t>(cur.r)) - kTwo23
                             : static_cast<float>(cur.r);
        const float lam = clamp ? 0.0f : rf * cur.inv_den_f;
        const bool gather = (flags & (is_col ? kGatherCols : kGatherRows)) != 0;
        const bool ident = (flags & (is_col ? kIdentityCols : kIdentityRows)) != 0;
        const int32_t first = __shfl_sync(0xffffffffu, i0, 0);
        const int32_t last = __shfl_sync(0xffffffffu, i1, 31);
        int32_t j0, j1, count;
        if (gather) {
            j0 = 2 * lane;
            j1 = 2 * lane + 1;
            int32_t *src_idx = is_col ? T.scol : T.srow;
            src_idx[j0] = i0;
            src_idx[j1] = i1;
            count = kMaxTile;
        } else {
            j0 = i0 - first;
            j1 = i1 - first;
            count = ident ? kBlock : last - first + 1;
        }
        if (is_col) {
            T.tx[0][lane] = j0;
            T.tx[1][lane] = j1;
            T.lx[lane] = lam;
        } else {
            T.ty[0][lane] = j0;
            T.ty[1][lane] = j1;
            T.ly[lane] = lam;
        }
        if (lane == 0) {
            if (is_col) {
                T.x_first = gather ? 0 : first;
                T.ncols = count;
                // chunks covering a row segment at any 16-byte offset: CQ <= 17 (C <= 4, count <= 64)
                const int CQ = (30 + C * count) >> 4;
                const int Q = (count + 3) >> 2;  // <= 16
                T.CQ = CQ;
                T.Q = Q;
                T.cmagic = kCeil65536[CQ];  // exact for x < 64 * 18
                T.qmagic = kCeil65536[Q];   // exact for x < 64 * 16
            } else {
                T.y_first = gather ? 0 : first;
                T.nrows = count;
            }
        }
    }
    if (!is_col && lane == 0) {
        T.flags = flags;
        T.W = W;
        T.C = C;
        T.gw2 = gw2;
        T.gh2 = Hr / kBlock;
        T.bh = bh;
        T.bw = bw;
        T.t = t;
        T.tt = tt;
        // a video half stages frame 2t + tt, the last frame standing in past the end
        const int64_t f = (flags & kVideo) ? min(2 * t + tt, D.frames - 1) : 0;
        T.src_off = D.src_off + f * D.frame_stride;
        T.limit = D.limit - f * D.frame_stride;
        T.row0 = D.row0;
        // merge order lists units by (t, block row, block col), column order by (t, block col, block row)
        const int gh2 = Hr / kBlock;
        const int64_t unit = static_cast<int64_t>(t) * gh2 * gw2 +
                             (P.order ? static_cast<int64_t>(bw) * gh2 + bh : static_cast<int64_t>(bh) * gw2 + bw);
        T.row_base = D.row0 + 4 * unit;
    }
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, int nbytes) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(src), "r"(nbytes) : "memory");
}

// Starts the asynchronous copy of block T's source row segments into the
// raw buffer: row j's bytes [rs, rs + C*ncols) are covered by 16-byte aligned
// chunks stored at raw + j*raw_stride. A chunk reaching past the caller's
// buffer is zero-filled there.
template <class Params>
__device__ __forceinline__ void issue_stage(const Params &P, const TapSet &T, uint8_t *raw, int tid) {
    const int flags = T.flags;
    if ((flags & kGatherCols) == 0) {
        const uint8_t *img = P.src + T.src_off;
        const int64_t limit = T.limit;
        const int W = T.W, C = T.C, CQ = T.CQ;
        const int y_first = T.y_first, x_first = T.x_first;
        const int L = C * T.ncols;
        const bool grow = (flags & kGatherRows) != 0;
        const int jobs = T.nrows * CQ;
        const uint32_t cmagic = T.cmagic;
        for (int job = tid; job < jobs; job += kThreads) {
            const int j = static_cast<int>((static_cast<uint32_t>(job) * cmagic) >> 16);
            const int c = job - j * CQ;
            const int sy = grow ? T.srow[j] : y_first + j;
            const int64_t rs = (static_cast<int64_t>(sy) * W + x_first) * C;
            const int64_t cs = (rs & ~int64_t(15)) + 16 * c;
            if (cs < rs + L) {
                const int64_t left = limit - cs;
                const int nb = left < 16 ? static_cast<int>(left) : 16;
                if (MIMO_CHECK(cs >= 0 && nb > 0 && cs + nb <= limit, kChkSrcCopy) &&
                    MIMO_CHECK(j < P.tile_rows && 16 * c + 16 <= P.raw_stride, kChkSmem))
                    cp_async16(raw + j * P.raw_stride + 16 * c, img + cs, nb);
            }
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// The two taps of one output column in a contiguously staged RGB row: the
// pixel at byte offset o in bytes 0..2 of `a`, and in bytes 0..2 of `b` the
// next pixel, or the same one again at the clamped right edge (`next` false).
// Three aligned 32-bit shared loads and funnel shifts.
__device__ __forceinline__ void rgb_pair(const uint8_t *row, uint32_t o, bool next, uint32_t &a, uint32_t &b) {
    const uint32_t *w = reinterpret_cast<const uint32_t *>(row + (o & ~3u));
    const uint32_t sh = (o & 3u) * 8u;
    const uint32_t w0 = w[0], w1 = w[1], w2 = w[2];
    a = __funnelshift_r(w0, w1, sh);
    const uint32_t hi = __funnelshift_r(w1, w2, sh);
    b = next ? __funnelshift_r(a, hi, 24) : a;
}

// Whether block T's staged rows are converted and interpolated along W in one
// step (RGB, resized width, contiguously staged columns); emit_block then
// skips its horizontal pass. Kernels instantiated without the fused step
// (kFused false: launches with no such image) never take it.
template <bool kFused>
__device__ __forceinline__ bool fused_hpass(const TapSet &T) {
    return kFused && T.C == 3 && (T.flags & (kIdentityCols | kGatherCols)) == 0;
}

// Converts block T's staged bytes to planar fp32 in the tile (RGBA
// composited onto white): a job = 4 consecutive pixels of one tile row.
// For RGB with a resized width a job is instead one quad of output columns of
// a tile row, interpolated along W on the way (fused_hpass). Gathered columns
// are loaded here directly from global memory.
template <bool kFused, class Params>
__device__ __forceinline__ void finish_stage(const Params &P, const TapSet &T, const uint8_t *raw, float *tile,
                                             int TS, int plane, int tid) {
    const int flags = T.flags;
    const int nrows = T.nrows;
    const int C = T.C;
    const float2 m23 = f2(-kTwo23, -kTwo23);
    if (fused_hpass<kFused>(T)) {
        // job = (tile row j, output column pair q): the two taps of each of the pair's output columns
        // come straight from the staged bytes, and (1 - lx) a + lx b = fma(lx, b - a, a) lands over
        // columns 2q, 2q+1 of the tile row. b - a is formed exactly from the 2^23 bit patterns, so the
        // values equal those of converting the row and then interpolating it. Pairs rather than quads:
        // the ~34 staged rows x 16 pairs fill three rounds of warps 2-7 evenly, where quads left a
        // second round on 80 of its 192 threads.
        const int W = T.W, y_first = T.y_first, x_first = T.x_first;
        const bool grow = (flags & kGatherRows) != 0;
        const int jobs = nrows * 16;
        const int t0 = (jobs <= 3 * (kThreads - 64)) ? 64 : 0;
        const int step = kThreads - t0;
        const float2 neg1 = f2(-1.0f, -1.0f);
        for (int job = tid - t0; job < jobs; job += step) {
            if (job < 0) break;
            const int j = job >> 4, q = job & 15;
            const int sy = grow ? T.srow[j] : y_first + j;
            const uint32_t mis = ((static_cast<uint32_t>(sy) * static_cast<uint32_t>(W) + x_first) * 3u) & 15u;
            const uint8_t *row = raw + j * P.raw_stride;
            const int2 ta = *reinterpret_cast<const int2 *>(&T.tx[0][2 * q]);
            const int2 tb = *reinterpret_cast<const int2 *>(&T.tx[1][2 * q]);
            const float2 l01 = *reinterpret_cast<const float2 *>(&T.lx[2 * q]);
            // every tap read (three words from the first tap) stays inside the staged row, every write
            // inside the tile, and the second tap is the first one or the pixel after it
            if (!MIMO_CHECK(j < P.tile_rows && 2 * q + 2 <= TS && min(ta.x, ta.y) >= 0 &&
                                static_cast<unsigned>(tb.x - ta.x) <= 1u && static_cast<unsigned>(tb.y - ta.y) <= 1u &&
                                ((mis + 3u * static_cast<uint32_t>(max(ta.x, ta.y))) & ~3u) + 12u <=
                                    static_cast<uint32_t>(P.raw_stride),
                            kChkSmem))
                continue;
            uint32_t a0, a1, b0, b1;
            rgb_pair(row, mis + 3u * ta.x, tb.x != ta.x, a0, b0);
            rgb_pair(row, mis + 3u * ta.y, tb.y != ta.y, a1, b1);
            float *t = tile + j * TS + 2 * q;
#define MIMO_FUSED_CHANNEL(c)                                                                                   \
    {                                                                                                           \
        const float2 A01 = f2(byte_bits<c>(a0), byte_bits<c>(a1));                                              \
        const float2 v01 = fma2(l01, fma2(A01, neg1, f2(byte_bits<c>(b0), byte_bits<c>(b1))), add2(A01, m23)); \
        *reinterpret_cast<float2 *>(t + (c) * plane) = v01;                                                     \
    }
            MIMO_FUSED_CHANNEL(0)
            MIMO_FUSED_CHANNEL(1)
            MIMO_FUSED_CHANNEL(2)
#undef MIMO_FUSED_CHANNEL
        }
    } else if ((flags & kGatherCols) == 0) {
        const int W = T.W, y_first = T.y_first, x_first = T.x_first;
        const bool grow = (flags & kGatherRows) != 0;
        const int Q = T.Q;
        const uint32_t qmagic = T.qmagic;
        const int jobs = nrows * Q;
        // warps 0-1 compute the next block's taps in this phase: leave them
        // out of the conversion unless the block has many jobs
        const int t0 = (jobs <= 2 * (kThreads - 64)) ? 64 : 0;
        const int step = kThreads - t0;
        for (int job = tid - t0; job < jobs; job += step) {
            if (job < 0) break;
            const int j = static_cast<int>((static_cast<uint32_t>(job) * qmagic) >> 16);
            const int px0 = (job - j * Q) * 4;
            const int sy = grow ? T.srow[j] : y_first + j;
            // low 4 bits of the row segment's byte offset (exact under 32-bit wraparound)
            const uint32_t mis = ((static_cast<uint32_t>(sy) * static_cast<uint32_t>(W) + x_first) *
                                  static_cast<uint32_t>(C)) & 15u;
            const uint32_t o = mis + static_cast<uint32_t>(C * px0);
            if (!MIMO_CHECK(j < P.tile_rows && px0 + 4 <= TS && (o & ~3u) + 16u <= static_cast<uint32_t>(P.raw_stride),
                            kChkSmem))
                continue;
            const uint32_t *rw = reinterpret_cast<const uint32_t *>(raw + j * P.raw_stride) + (o >> 2);
            const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2], w3 = rw[3];
            float2 R0, R1, G0, G1, B0, B1;
            if (C == 4) {
                // o is a multiple of 4: 4 whole RGBA pixels; white = 65025 - 255 a
                const float2 A01 = add2(f2(byte_bits<3>(w0), byte_bits<3>(w1)), m23);
                const float2 A23 = add2(f2(byte_bits<3>(w2), byte_bits<3>(w3)), m23);
                const float2 wh01 = fma2(A01, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
                const float2 wh23 = fma2(A23, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
                R0 = on_white2(add2(f2(byte_bits<0>(w0), byte_bits<0>(w1)), m23), A01, wh01);
                R1 = on_white2(add2(f2(byte_bits<0>(w2), byte_bits<0>(w3)), m23), A23, wh23);
                G0 = on_white2(add2(f2(byte_bits<1>(w0), byte_bits<1>(w1)), m23), A01, wh01);
                G1 = on_white2(add2(f2(byte_bits<1>(w2), byte_bits<1>(w3)), m23), A23, wh23);
                B0 = on_white2(add2(f2(byte_bits<2>(w0), byte_bits<2>(w1)), m23), A01, wh01);
                B1 = on_white2(add2(f2(byte_bits<2>(w2), byte_bits<2>(w3)), m23), A23, wh23);
            } else {
                // 12 bytes from o, realigned by the byte offset within the word
                const int sh = static_cast<int>(o & 3u) * 8;
                const uint32_t r0 = __funnelshift_r(w0, w1, sh);
                const uint32_t r1 = __funnelshift_r(w1, w2, sh);
                const uint32_t r2 = __funnelshift_r(w2, w3, sh);
                // bytes: r0 = R0 G0 B0 R1 | r1 = G1 B1 R2 G2 | r2 = B2 R3 G3 B3
                R0 = add2(f2(byte_bits<0>(r0), byte_bits<3>(r0)), m23);
                R1 = add2(f2(byte_bits<2>(r1), byte_bits<1>(r2)), m23);
                G0 = add2(f2(byte_bits<1>(r0), byte_bits<0>(r1)), m23);
                G1 = add2(f2(byte_bits<3>(r1), byte_bits<2>(r2)), m23);
                B0 = add2(f2(byte_bits<2>(r0), byte_bits<1>(r1)), m23);
                B1 = add2(f2(byte_bits<0>(r2), byte_bits<3>(r2)), m23);
            }
            float *t = tile + j * TS + px0;
            *reinterpret_cast<float4 *>(t) = make_float4(R0.x, R0.y, R1.x, R1.y);
            *reinterpret_cast<float4 *>(t + plane) = make_float4(G0.x, G0.y, G1.x, G1.y);
            *reinterpret_cast<float4 *>(t + 2 * plane) = make_float4(B0.x, B0.y, B1.x, B1.y);
        }
    } else {
        const uint8_t *img = P.src + T.src_off;
        const int64_t W = T.W;
        const bool grow = (flags & kGatherRows) != 0;
        const int total = nrows * kMaxTile;
        for (int e = tid; e < total; e += kThreads) {
            const int j = e >> 6;
            const int i = e & (kMaxTile - 1);
            const int sy = grow ? T.srow[j] : T.y_first + j;
            const int64_t pix = static_cast<int64_t>(sy) * W + T.scol[i];
            if (!MIMO_CHECK(pix >= 0 && (pix + 1) * C <= T.limit && j < P.tile_rows && i < TS, kChkSrcLoad)) continue;
            float r, g, b;
            if (C == 4) {
                const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(img) + pix);
                const float a = byte_f<3>(v);
                const float wh = fmaf(a, -255.0f, 65025.0f);
                const float2 rg = on_white2(add2(f2(byte_bits<0>(v), byte_bits<1>(v)), m23), f2(a, a), f2(wh, wh));
                const float2 bx = on_white2(add2(f2(byte_bits<2>(v), byte_bits<2>(v)), m23), f2(a, a), f2(wh, wh));
                r = rg.x;
                g = rg.y;
                b = bx.x;
            } else {
                const uint8_t *px = img + 3 * pix;
                r = static_cast<float>(__ldg(px));
                g = static_cast<float>(__ldg(px + 1));
                b = static_cast<float>(__ldg(px + 2));
            }
            float *t = tile + j * TS + i;
            t[0] = r;
            t[plane] = g;
            t[2 * plane] = b;
        }
    }
}

// Normalises one channel's 4 interpolated values (x*k + b) and stores them at
// column `col` of output row `row`: into both temporal slots for an image
// (`both`), into the slot at `slot0` for a video half. Streaming stores.
template <bool kBF16, class Params>
__device__ __forceinline__ void store_quad(const Params &P, int64_t row, int c, int col, int slot0, bool both,
                                           float2 v01, float2 v23) {
    if (!MIMO_CHECK(row >= P.chk_row_lo && row < P.chk_row_hi, kChkRowStore)) return;
    const float2 k2 = f2(P.k[c], P.k[c]), b2 = f2(P.b[c], P.b[c]);
    const float2 n01 = fma2(v01, k2, b2);
    const float2 n23 = fma2(v23, k2, b2);
    if constexpr (!kBF16) {
        float *o = static_cast<float *>(P.out) + row * kRowWidth + c * 512 + col + slot0;
        const float4 f4 = make_float4(n01.x, n01.y, n23.x, n23.y);
        __stcs(reinterpret_cast<float4 *>(o), f4);
        if (both) __stcs(reinterpret_cast<float4 *>(o + 256), f4);
    } else {
        __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(P.out) + row * kRowWidth + c * 512 + col + slot0;
        const __nv_bfloat162 lo2 = __floats2bfloat162_rn(n01.x, n01.y);
        const __nv_bfloat162 hi2 = __floats2bfloat162_rn(n23.x, n23.y);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&lo2);
        u.y = *reinterpret_cast<const uint32_t *>(&hi2);
        if (P.keep_rows) {
            // rows that the patch embedding reads right after this launch (mimo_preprocess_embed): stored
            // with an L2 evict-last policy so that they are read back from L2, not from HBM
            uint64_t pol;
            asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
            asm volatile("st.global.L2::cache_hint.v2.b32 [%0], {%1, %2}, %3;" ::"l"(o), "r"(u.x), "r"(u.y), "l"(pol)
                         : "memory");
            if (both)
                asm volatile("st.global.L2::cache_hint.v2.b32 [%0], {%1, %2}, %3;" ::"l"(o + 256), "r"(u.x), "r"(u.y),
                             "l"(pol)
                             : "memory");
        } else {
            __stcs(reinterpret_cast<uint2 *>(o), u);
            if (both) __stcs(reinterpret_cast<uint2 *>(o + 256), u);
        }
    }
}

// The merge unit's table entries, written by threads 0-2 of the block: the
// column-order permutation (thread 0), the rotary positions of the unit's 4
// emitted rows starting at `row_base` (thread 1), the window index (thread 2).
// `row0` is the item's first row, `t_units` the units of its earlier temporal
// patches.
template <class Params>
__device__ __forceinline__ void write_unit_tables(const Params &P, int tid, int64_t row0, int64_t t_units, int bh,
                                                  int bw, int gh2, int gw2, int64_t row_base) {
    const int64_t src_unit = t_units + static_cast<int64_t>(bh) * gw2 + bw;  // merge order
    const int64_t dst_unit = t_units + static_cast<int64_t>(bw) * gh2 + bh;  // column order
    if (tid == 0 && P.perm != nullptr) {
        const int32_t s0 = static_cast<int32_t>(row0 + 4 * src_unit);
        if (MIMO_CHECK(row0 + 4 * dst_unit >= 0 && row0 + 4 * dst_unit + 4 <= P.chk_table_rows, kChkTableStore))
            __stcs(reinterpret_cast<int4 *>(P.perm + row0 + 4 * dst_unit), make_int4(s0, s0 + 1, s0 + 2, s0 + 3));
    } else if (tid == 1 && P.pos != nullptr) {
        // rows (mh, mw) = (0,0), (0,1), (1,0), (1,1) of the unit
        const int32_t h = 2 * bh, w = 2 * bw;
        int4 *d = reinterpret_cast<int4 *>(P.pos + 2 * row_base);
        if (MIMO_CHECK(row_base >= P.chk_row_lo && row_base + 4 <= P.chk_row_hi, kChkTableStore)) {
            __stcs(d, make_int4(h, w, h, w + 1));
            __stcs(d + 1, make_int4(h + 1, w, h + 1, w + 1));
        }
    } else if (tid == 2 && P.win != nullptr) {
        const int64_t u0 = row0 / 4;
        if (MIMO_CHECK(u0 + dst_unit >= 0 && 4 * (u0 + dst_unit) + 4 <= P.chk_table_rows, kChkTableStore))
            P.win[u0 + dst_unit] = static_cast<int32_t>(u0 + src_unit);
    }
}

// Interpolation, normalisation and stores of one staged block.
template <bool kBF16, bool kFused, class Params>
__device__ __forceinline__ void emit_block(const Params &P, const TapSet &T, float *tile, int TS, int plane,
                                           int tid, int warp, int lane) {
    const int flags = T.flags;
    const int nrows = T.nrows;

    // horizontal pass (resized widths only), in place: the warp owning tile
    // row j reads every lane's two taps, then writes the 32 interpolated
    // values over columns 0..31 of the same row
    const bool hpass = (flags & kIdentityCols) == 0 && !fused_hpass<kFused>(T);
    if (hpass) {
        const int x0 = T.tx[0][lane], x1 = T.tx[1][lane];
        const float lx = T.lx[lane];
        for (int j = warp; j < nrows; j += kThreads / 32) {
            float *t = tile + j * TS;
            float h[3];
            // a lane whose check fails skips its accesses, never the __syncwarp
            const bool ok = MIMO_CHECK(j < P.tile_rows && x0 >= 0 && x1 >= 0 && x0 < TS && x1 < TS, kChkSmem);
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                const float a = ok ? t[c * plane + x0] : 0.0f;
                const float b = ok ? t[c * plane + x1] : 0.0f;
                h[c] = fmaf(lx, b - a, a);
            }
            __syncwarp();
            if (ok) {
#pragma unroll
                for (int c = 0; c < 3; ++c) t[c * plane + lane] = h[c];
            }
        }
        __syncthreads();
    }

    // vertical pass + normalisation + both temporal copies. Warp w covers
    // output rows dy = 4w..4w+3 of the block; a lane covers 4 consecutive
    // columns. For fixed mw the 16 lanes write 4 consecutive 16-float
    // segments of one output row: 256 contiguous bytes (fp32).
    const int mh = warp >> 2;
    const int py = ((warp & 3) << 2) | (lane >> 3);
    const int mw = (lane >> 2) & 1;
    const int q = lane & 3;
    const int dy = (mh << 4) | py;
    const int dx0 = (mw << 4) | (q << 2);
    const bool yident = (flags & kIdentityRows) != 0;
    if (!MIMO_CHECK(T.ty[0][dy] >= 0 && T.ty[1][dy] >= 0 && T.ty[0][dy] < P.tile_rows && T.ty[1][dy] < P.tile_rows &&
                        dx0 + 4 <= TS,
                    kChkSmem))
        return;
    const float *a_row = tile + T.ty[0][dy] * TS + dx0;
    const float *b_row = tile + T.ty[1][dy] * TS + dx0;
    // (1 - ly) a + ly b as two FMAs: a - ly a, then + ly b
    const float ly = T.ly[dy];
    const float2 ly2 = f2(ly, ly), nly2 = f2(-ly, -ly);
    const int64_t row = T.row_base + (mh * 2 + mw);
    const int col = py * 16 + q * 4;
    const bool video = (flags & kVideo) != 0;
    const bool both = !video;
    const int slot0 = video ? 256 * T.tt : 0;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        const float4 A = *reinterpret_cast<const float4 *>(a_row + c * plane);
        float2 v01 = f2(A.x, A.y), v23 = f2(A.z, A.w);
        if (!yident) {
            const float4 B = *reinterpret_cast<const float4 *>(b_row + c * plane);
            v01 = fma2(ly2, f2(B.x, B.y), fma2(nly2, v01, v01));
            v23 = fma2(ly2, f2(B.z, B.w), fma2(nly2, v23, v23));
        }
        // an image fills both temporal slots with its one frame; a video half fills slot tt
        store_quad<kBF16>(P, row, c, col, slot0, both, v01, v23);
    }

    // the merge unit's table entries (once per unit: a video's tt = 0 half)
    if (tid < 3 && (!video || T.tt == 0))
        write_unit_tables(P, tid, T.row0, static_cast<int64_t>(T.t) * T.gh2 * T.gw2, T.bh, T.bw, T.gh2, T.gw2,
                          T.row_base);
}

// Persistent CTAs: CTA c takes the contiguous block range
// [c*B/G, (c+1)*B/G) of the launch and pipelines it. While block k is
// interpolated and stored, the source bytes of block k+1 are already in
// shared memory and those of block k+2 are in flight (cp.async), and warps
// 0-1 compute the taps of the block after.
template <bool kBF16, bool kFused, class Params>
__global__ void __launch_bounds__(kThreads, 5) preprocess_kernel(const __grid_constant__ Params P) {
    extern __shared__ float4 smem4[];
    float *const tile = reinterpret_cast<float *>(smem4);  // [3][rows][stride] | raw bytes
    uint8_t *const raw = reinterpret_cast<uint8_t *>(tile + P.raw);
    __shared__ TapSet S[2];
    __shared__ AxisCursor s_cur[64];  // one per lane of the two tap warps

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int TS = P.tile_stride;
    const int plane = P.tile_rows * TS;
    const int64_t B = P.block_start[P.n];
    const int begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * B / gridDim.x);
    const int end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * B / gridDim.x);
    if (begin >= end) return;

    AxisCursor &cur = s_cur[tid & 63];  // meaningful for warps 0-1 only
    if (warp < 2) {
        cur = AxisCursor();
        compute_taps(P, S[0], S[1], begin, cur, warp, lane);
    }
    __syncthreads();
    if (warp < 2 && begin + 1 < end) compute_taps(P, S[1], S[0], begin + 1, cur, warp, lane);
    issue_stage(P, S[0], raw, tid);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    finish_stage<kFused>(P, S[0], raw, tile, TS, plane, tid);
    __syncthreads();
    if (begin + 1 < end) issue_stage(P, S[1], raw, tid);

    int slot = 0;
    for (int blk = begin; blk < end; ++blk) {
        emit_block<kBF16, kFused>(P, S[slot], tile, TS, plane, tid, warp, lane);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();  // tile and S[slot] free; raw holds block blk+1
        if (blk + 1 < end) finish_stage<kFused>(P, S[slot ^ 1], raw, tile, TS, plane, tid);
        if (warp < 2 && blk + 2 < end) compute_taps(P, S[slot], S[slot ^ 1], blk + 2, cur, warp, lane);
        __syncthreads();  // tile holds block blk+1, S[slot] the taps of blk+2, raw is free
        if (blk + 2 < end) issue_stage(P, S[slot], raw, tid);
        slot ^= 1;
    }
}

// ---------------------------------------------------------------------------
// Direct kernel, for launches whose images (or video frames) all keep their
// width (Wr == W). Every output column then samples its own source column, and
// a block needs no staging. Each thread owns the same 4 pixels x 3 channels of
// one output row in every block, as in the staged kernel's vertical pass. It
// reads its one or two source rows straight from global memory (the ~2x reuse
// between neighbouring output rows hits L1), converts the bytes with the
// staged kernel's arithmetic, and then interpolates, normalises and stores
// identically. There is no shared memory and no barrier. The row taps come
// from the exact quotient, once per block row, and stay in registers. Each
// row quad is one 16-byte load (RGBA) or three 4-byte loads (RGB).
// bf16 rows take another mapping (direct_bf16x8): each half of the CTA takes
// every other block, and a thread owns 8 consecutive pixels of one output row,
// so each channel leaves in one 16-byte store per temporal slot instead of two
// 8-byte ones, and the per-block work is spread over twice the pixels.
// ---------------------------------------------------------------------------

// The 4-pixel quad a thread reads from one source row. Every width on this
// path is a multiple of 32 (Wr == W) and a thread's first column a multiple of
// 4, so an RGB quad (12 bytes) starts 4-byte aligned and an RGBA quad (16
// bytes) 16-byte aligned, both wholly inside the image (image offsets are
// 16-byte aligned).
__device__ __forceinline__ void load_quad(const uint8_t *p, int C, uint32_t (&w)[4]) {
    if (C == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
    } else {
        const uint32_t *q = reinterpret_cast<const uint32_t *>(p);
        w[0] = __ldg(q);
        w[1] = __ldg(q + 1);
        w[2] = __ldg(q + 2);
        w[3] = 0u;
    }
}

// The quad as planar floats on 0..255 (RGBA composited onto white), with
// finish_stage's arithmetic.
__device__ __forceinline__ void convert4(const uint32_t (&w)[4], int C, float4 (&v)[3]) {
    const float2 m23 = f2(-kTwo23, -kTwo23);
    float2 R0, R1, G0, G1, B0, B1;
    if (C == 4) {
        const float2 A01 = add2(f2(byte_bits<3>(w[0]), byte_bits<3>(w[1])), m23);
        const float2 A23 = add2(f2(byte_bits<3>(w[2]), byte_bits<3>(w[3])), m23);
        const float2 wh01 = fma2(A01, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
        const float2 wh23 = fma2(A23, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
        R0 = on_white2(add2(f2(byte_bits<0>(w[0]), byte_bits<0>(w[1])), m23), A01, wh01);
        R1 = on_white2(add2(f2(byte_bits<0>(w[2]), byte_bits<0>(w[3])), m23), A23, wh23);
        G0 = on_white2(add2(f2(byte_bits<1>(w[0]), byte_bits<1>(w[1])), m23), A01, wh01);
        G1 = on_white2(add2(f2(byte_bits<1>(w[2]), byte_bits<1>(w[3])), m23), A23, wh23);
        B0 = on_white2(add2(f2(byte_bits<2>(w[0]), byte_bits<2>(w[1])), m23), A01, wh01);
        B1 = on_white2(add2(f2(byte_bits<2>(w[2]), byte_bits<2>(w[3])), m23), A23, wh23);
    } else {
        // bytes: w0 = R0 G0 B0 R1 | w1 = G1 B1 R2 G2 | w2 = B2 R3 G3 B3
        R0 = add2(f2(byte_bits<0>(w[0]), byte_bits<3>(w[0])), m23);
        R1 = add2(f2(byte_bits<2>(w[1]), byte_bits<1>(w[2])), m23);
        G0 = add2(f2(byte_bits<1>(w[0]), byte_bits<0>(w[1])), m23);
        G1 = add2(f2(byte_bits<3>(w[1]), byte_bits<2>(w[2])), m23);
        B0 = add2(f2(byte_bits<2>(w[0]), byte_bits<1>(w[1])), m23);
        B1 = add2(f2(byte_bits<0>(w[2]), byte_bits<3>(w[2])), m23);
    }
    v[0] = make_float4(R0.x, R0.y, R1.x, R1.y);
    v[1] = make_float4(G0.x, G0.y, G1.x, G1.y);
    v[2] = make_float4(B0.x, B0.y, B1.x, B1.y);
}

// The direct kernel's bf16 rows: each half of the CTA (128 threads) takes
// every other block of the CTA's range, and a thread owns 8 consecutive pixels
// of one output row of its block, so each channel's 8 bf16 values leave in one
// 16-byte store per temporal slot, and its two source rows arrive in a few wide
// loads issued together. Per pixel the arithmetic is that of the fp32 path
// below, quad by quad, then the same round to bf16.
template <bool kVideoLaunch, class Params>
__device__ __forceinline__ void direct_bf16x8(const Params &P) {
    const int tid = threadIdx.x;
    const int grp = tid >> 7, g = tid & 127;
    const int w4 = g >> 5, lane = tid & 31;
    const int64_t B = P.block_start[P.n];
    const int begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * B / gridDim.x);
    const int end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * B / gridDim.x);
    const int first = begin + grp;
    if (first >= end) return;

    // this thread's place in every block: warp w4 of the half covers output rows 8 (w4 & 1) .. +7 of
    // patch row mh = w4 >> 1; for each mw, 16 lanes write 256 contiguous bytes of an output row
    const int mh = w4 >> 1;
    const int py = ((w4 & 1) << 3) | (lane >> 2);
    const int mw = (lane >> 1) & 1;
    const int q2 = lane & 1;
    const int dy = (mh << 4) | py;
    const int dx0 = (mw << 4) | (q2 << 3);
    const int col = py * 16 + q2 * 8;

    int ii = find_image(P, first);
    int t, bh, bw, tt;
    {
        const ImageDesc &D = P.img[ii];
        const int gq = D.Wr / kBlock;
        int local = first - P.block_start[ii] + (ii == 0 ? P.unit0 : 0);
        const bool vid = (D.flags & kVideo) != 0;
        tt = vid ? (local & 1) : 0;
        if (vid) local >>= 1;
        const int units = (D.Hr / kBlock) * gq;
        t = local / units;
        local -= t * units;
        bh = local / gq;
        bw = local - bh * gq;
    }
    // one block on: the other temporal slot of a video's unit, else one column on, then the next block
    // row, then the next temporal patch (a video) or image
    auto advance = [&]() {
        const ImageDesc &Dn = P.img[ii];
        const int g_w = Dn.Wr / kBlock, g_h = Dn.Hr / kBlock;
        if constexpr (kVideoLaunch) {
            if (tt == 0) {
                tt = 1;
            } else {
                tt = 0;
                if (++bw == g_w) {
                    bw = 0;
                    if (++bh == g_h) {
                        bh = 0;
                        ++t;
                    }
                }
            }
        } else {
            if (++bw == g_w) {
                bw = 0;
                if (++bh == g_h) {
                    bh = 0;
                    ++ii;
                }
            }
        }
    };
    int tap_ii = -1, tap_bh = -1;
    int32_t sy0 = 0, sy1 = 0;
    float ly = 0.0f;
    for (int blk = first; blk < end; blk += 2) {
        const ImageDesc &D = P.img[ii];
        const int32_t H = D.H, W = D.W, Hr = D.Hr, flags = D.flags;
        const int C = (flags >> kChannelShift) & 0xFF;
        const bool yident = (flags & kIdentityRows) != 0;
        if (ii != tap_ii || bh != tap_bh) {
            const int64_t den = 2 * static_cast<int64_t>(Hr);
            const double inv_den = 1.0 / static_cast<double>(den);
            const int64_t Y = static_cast<int64_t>(bh) * kBlock + dy;
            const int64_t num = (2 * Y + 1) * H - Hr;
            int64_t qq = static_cast<int64_t>(floor(static_cast<double>(num) * inv_den));
            int64_t r = num - qq * den;
            while (r < 0) {
                --qq;
                r += den;
            }
            while (r >= den) {
                ++qq;
                r -= den;
            }
            const bool clamp = qq < 0;
            sy0 = clamp ? 0 : static_cast<int32_t>(qq);
            sy1 = (static_cast<int64_t>(sy0) + 1 < H) ? sy0 + 1 : H - 1;
            ly = clamp ? 0.0f : static_cast<float>(r) * static_cast<float>(inv_den);
            tap_ii = ii;
            tap_bh = bh;
        }
        const bool video = kVideoLaunch;
        const int64_t f = video ? min(2 * t + tt, D.frames - 1) : 0;
        const uint8_t *img = P.src + D.src_off + f * D.frame_stride;
        [[maybe_unused]] const int64_t frame_bytes = static_cast<int64_t>(H) * W * C;
        const float2 ly2 = f2(ly, ly), nly2 = f2(-ly, -ly);
        uint32_t pk[3][4];  // channel c: bf16 pairs of pixels (0,1), (2,3), (4,5), (6,7)
        // the loads of both quads of both rows go out before any conversion. RGBA: the 8 pixels of a row
        // are 32 bytes at a 16-byte boundary, two 16-byte loads. RGB: 24 bytes at an 8-byte boundary
        // (W a multiple of 32, the first column of 8, the frame 16-byte aligned), three 8-byte loads
        uint2 ra[3] = {make_uint2(0u, 0u), make_uint2(0u, 0u), make_uint2(0u, 0u)};
        uint2 rb[3] = {make_uint2(0u, 0u), make_uint2(0u, 0u), make_uint2(0u, 0u)};
        uint4 qa4[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
        uint4 qb4[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
        if (C == 4) {
            const int64_t x0 = static_cast<int64_t>(bw) * kBlock + dx0;
            const int64_t pa = (static_cast<int64_t>(sy0) * W + x0) * 4, pb = (static_cast<int64_t>(sy1) * W + x0) * 4;
            if (MIMO_CHECK(pa >= 0 && pa + 32 <= frame_bytes && f * D.frame_stride + pa + 32 <= D.limit &&
                               (reinterpret_cast<uintptr_t>(img + pa) & 15u) == 0,
                           kChkSrcLoad)) {
                qa4[0] = __ldg(reinterpret_cast<const uint4 *>(img + pa));
                qa4[1] = __ldg(reinterpret_cast<const uint4 *>(img + pa) + 1);
            }
            if (!yident && MIMO_CHECK(pb >= 0 && pb + 32 <= frame_bytes && f * D.frame_stride + pb + 32 <= D.limit &&
                                          (reinterpret_cast<uintptr_t>(img + pb) & 15u) == 0,
                                      kChkSrcLoad)) {
                qb4[0] = __ldg(reinterpret_cast<const uint4 *>(img + pb));
                qb4[1] = __ldg(reinterpret_cast<const uint4 *>(img + pb) + 1);
            }
        } else {
            const int64_t x0 = static_cast<int64_t>(bw) * kBlock + dx0;
            const int64_t pa = (static_cast<int64_t>(sy0) * W + x0) * 3, pb = (static_cast<int64_t>(sy1) * W + x0) * 3;
            if (MIMO_CHECK(pa >= 0 && pa + 24 <= frame_bytes && f * D.frame_stride + pa + 24 <= D.limit &&
                               (reinterpret_cast<uintptr_t>(img + pa) & 7u) == 0,
                           kChkSrcLoad)) {
                const uint2 *q = reinterpret_cast<const uint2 *>(img + pa);
                ra[0] = __ldg(q);
                ra[1] = __ldg(q + 1);
                ra[2] = __ldg(q + 2);
            }
            if (!yident && MIMO_CHECK(pb >= 0 && pb + 24 <= frame_bytes && f * D.frame_stride + pb + 24 <= D.limit &&
                                          (reinterpret_cast<uintptr_t>(img + pb) & 7u) == 0,
                                      kChkSrcLoad)) {
                const uint2 *q = reinterpret_cast<const uint2 *>(img + pb);
                rb[0] = __ldg(q);
                rb[1] = __ldg(q + 1);
                rb[2] = __ldg(q + 2);
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t wa[4] = {0u, 0u, 0u, 0u}, wb[4] = {0u, 0u, 0u, 0u};
            float4 va[3], vb[3];
            if (C == 3) {
                // words 3h .. 3h+2 of the row's six
                wa[0] = h ? ra[1].y : ra[0].x;
                wa[1] = h ? ra[2].x : ra[0].y;
                wa[2] = h ? ra[2].y : ra[1].x;
                wb[0] = h ? rb[1].y : rb[0].x;
                wb[1] = h ? rb[2].x : rb[0].y;
                wb[2] = h ? rb[2].y : rb[1].x;
            } else {
                const uint4 a4 = h ? qa4[1] : qa4[0], b4 = h ? qb4[1] : qb4[0];
                wa[0] = a4.x;
                wa[1] = a4.y;
                wa[2] = a4.z;
                wa[3] = a4.w;
                wb[0] = b4.x;
                wb[1] = b4.y;
                wb[2] = b4.z;
                wb[3] = b4.w;
            }
            if (!yident) convert4(wb, C, vb);
            convert4(wa, C, va);
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                float2 v01 = f2(va[c].x, va[c].y), v23 = f2(va[c].z, va[c].w);
                if (!yident) {
                    v01 = fma2(ly2, f2(vb[c].x, vb[c].y), fma2(nly2, v01, v01));
                    v23 = fma2(ly2, f2(vb[c].z, vb[c].w), fma2(nly2, v23, v23));
                }
                const float2 k2 = f2(P.k[c], P.k[c]), b2 = f2(P.b[c], P.b[c]);
                const float2 n01 = fma2(v01, k2, b2);
                const float2 n23 = fma2(v23, k2, b2);
                const __nv_bfloat162 lo2 = __floats2bfloat162_rn(n01.x, n01.y);
                const __nv_bfloat162 hi2 = __floats2bfloat162_rn(n23.x, n23.y);
                pk[c][2 * h] = *reinterpret_cast<const uint32_t *>(&lo2);
                pk[c][2 * h + 1] = *reinterpret_cast<const uint32_t *>(&hi2);
            }
        }
        const int gw2 = D.Wr / kBlock, gh2 = Hr / kBlock;
        const int64_t t_units = static_cast<int64_t>(t) * gh2 * gw2;
        const int64_t unit =
            t_units + (P.order ? static_cast<int64_t>(bw) * gh2 + bh : static_cast<int64_t>(bh) * gw2 + bw);
        const int64_t row = D.row0 + 4 * unit + (mh * 2 + mw);
        const int slot0 = video ? 256 * tt : 0;
        if (MIMO_CHECK(row >= P.chk_row_lo && row < P.chk_row_hi, kChkRowStore)) {
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(P.out) + row * kRowWidth + c * 512 + col + slot0;
                const uint4 u = make_uint4(pk[c][0], pk[c][1], pk[c][2], pk[c][3]);
                if (P.keep_rows) {
                    uint64_t pol;
                    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
                    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(o), "r"(u.x),
                                 "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol)
                                 : "memory");
                    if (!video)
                        asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(o + 256),
                                     "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol)
                                     : "memory");
                } else {
                    __stcs(reinterpret_cast<uint4 *>(o), u);
                    if (!video) __stcs(reinterpret_cast<uint4 *>(o + 256), u);
                }
            }
        }
        if (g < 3 && (!video || tt == 0)) {
            const int64_t src_unit = t_units + static_cast<int64_t>(bh) * gw2 + bw;  // merge order
            const int64_t dst_unit = t_units + static_cast<int64_t>(bw) * gh2 + bh;  // column order
            if (g == 0 && P.perm != nullptr) {
                const int32_t s0 = static_cast<int32_t>(D.row0 + 4 * src_unit);
                if (MIMO_CHECK(D.row0 + 4 * dst_unit >= 0 && D.row0 + 4 * dst_unit + 4 <= P.chk_table_rows,
                               kChkTableStore))
                    __stcs(reinterpret_cast<int4 *>(P.perm + D.row0 + 4 * dst_unit),
                           make_int4(s0, s0 + 1, s0 + 2, s0 + 3));
            } else if (g == 1 && P.pos != nullptr) {
                const int32_t hh = 2 * bh, ww = 2 * bw;
                int4 *d = reinterpret_cast<int4 *>(P.pos + 2 * (D.row0 + 4 * unit));
                if (MIMO_CHECK(D.row0 + 4 * unit >= P.chk_row_lo && D.row0 + 4 * unit + 4 <= P.chk_row_hi,
                               kChkTableStore)) {
                    __stcs(d, make_int4(hh, ww, hh, ww + 1));
                    __stcs(d + 1, make_int4(hh + 1, ww, hh + 1, ww + 1));
                }
            } else if (g == 2 && P.win != nullptr) {
                const int64_t u0 = D.row0 / 4;
                if (MIMO_CHECK(u0 + dst_unit >= 0 && 4 * (u0 + dst_unit) + 4 <= P.chk_table_rows, kChkTableStore))
                    P.win[u0 + dst_unit] = static_cast<int32_t>(u0 + src_unit);
            }
        }
        if (blk + 2 < end) {
            advance();
            advance();
        }
    }
}

// bf16 rows need 64 registers for their two quads (4 CTAs per SM); fp32 rows
// keep 48 (a video) or 40 (images).
template <bool kBF16, bool kVideoLaunch, class Params>
__global__ void __launch_bounds__(kThreads, kBF16 ? 4 : (kVideoLaunch ? 5 : 6)) direct_kernel(
    const __grid_constant__ Params P) {
    if constexpr (kBF16) {
        direct_bf16x8<kVideoLaunch>(P);
        return;
    }
    // fp32 rows: 4 pixels per thread
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t B = P.block_start[P.n];
    const int begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * B / gridDim.x);
    const int end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * B / gridDim.x);
    if (begin >= end) return;

    // this thread's place in every block (the staged kernel's vertical-pass mapping)
    const int mh = warp >> 2;
    const int py = ((warp & 3) << 2) | (lane >> 3);
    const int mw = (lane >> 2) & 1;
    const int q = lane & 3;
    const int dy = (mh << 4) | py;
    const int dx0 = (mw << 4) | (q << 2);
    const int col = py * 16 + q * 4;

    // position of the first block (a video's blocks are (t, block row, block col, tt) halves, tt
    // innermost); later blocks advance one step at a time
    int ii = find_image(P, begin);
    int t, bh, bw, tt;
    {
        const ImageDesc &D = P.img[ii];
        const int g = D.Wr / kBlock;
        int local = begin - P.block_start[ii] + (ii == 0 ? P.unit0 : 0);
        const bool vid = (D.flags & kVideo) != 0;
        tt = vid ? (local & 1) : 0;
        if (vid) local >>= 1;
        const int units = (D.Hr / kBlock) * g;
        t = local / units;
        local -= t * units;
        bh = local / g;
        bw = local - bh * g;
    }
    int tap_ii = -1, tap_bh = -1;
    int32_t sy0 = 0, sy1 = 0;
    float ly = 0.0f;
    for (int blk = begin; blk < end; ++blk) {
        const ImageDesc &D = P.img[ii];
        const int32_t H = D.H, W = D.W, Hr = D.Hr, flags = D.flags;
        const int C = (flags >> kChannelShift) & 0xFF;
        const bool yident = (flags & kIdentityRows) != 0;
        if (ii != tap_ii || bh != tap_bh) {
            // exact taps of output row Y: i0 = floor(((2Y+1)*H - Hr) / (2*Hr)) clamped at 0,
            // i1 = min(i0+1, H-1), weight = remainder / (2*Hr); compute_taps reaches the same
            // quotient incrementally
            const int64_t den = 2 * static_cast<int64_t>(Hr);
            const double inv_den = 1.0 / static_cast<double>(den);
            const int64_t Y = static_cast<int64_t>(bh) * kBlock + dy;
            const int64_t num = (2 * Y + 1) * H - Hr;
            int64_t qq = static_cast<int64_t>(floor(static_cast<double>(num) * inv_den));
            int64_t r = num - qq * den;
            while (r < 0) {
                --qq;
                r += den;
            }
            while (r >= den) {
                ++qq;
                r -= den;
            }
            const bool clamp = qq < 0;
            sy0 = clamp ? 0 : static_cast<int32_t>(qq);
            sy1 = (static_cast<int64_t>(sy0) + 1 < H) ? sy0 + 1 : H - 1;
            ly = clamp ? 0.0f : static_cast<float>(r) * static_cast<float>(inv_den);
            tap_ii = ii;
            tap_bh = bh;
        }
        // a launch holds images only, or one video (kVideoLaunch): the image code carries no video work
        const bool video = kVideoLaunch;
        // a video half reads frame 2t + tt, the last frame standing in past the end
        const int64_t f = video ? min(2 * t + tt, D.frames - 1) : 0;
        const uint8_t *img = P.src + D.src_off + f * D.frame_stride;
        const int64_t x = static_cast<int64_t>(bw) * kBlock + dx0;
        uint32_t wa[4] = {0u, 0u, 0u, 0u}, wb[4] = {0u, 0u, 0u, 0u};
        float4 va[3], vb[3];
        // the quad's bytes lie inside the frame and the caller's buffer (skipped otherwise; the
        // checks, and with them frame_bytes, exist only in the bounds-checked build)
        [[maybe_unused]] const int64_t frame_bytes = static_cast<int64_t>(H) * W * C;
        const int64_t qa = (static_cast<int64_t>(sy0) * W + x) * C, qb = (static_cast<int64_t>(sy1) * W + x) * C;
        if (MIMO_CHECK(qa >= 0 && qa + (C == 4 ? 16 : 12) <= frame_bytes &&
                           f * D.frame_stride + qa + (C == 4 ? 16 : 12) <= D.limit,
                       kChkSrcLoad))
            load_quad(img + qa, C, wa);
        if (!yident) {
            if (MIMO_CHECK(qb >= 0 && qb + (C == 4 ? 16 : 12) <= frame_bytes &&
                               f * D.frame_stride + qb + (C == 4 ? 16 : 12) <= D.limit,
                           kChkSrcLoad))
                load_quad(img + qb, C, wb);
            convert4(wb, C, vb);
        }
        convert4(wa, C, va);

        // merge order lists units by (t, block row, block col), column order by (t, block col, block row)
        const int gw2 = D.Wr / kBlock, gh2 = Hr / kBlock;
        const int64_t t_units = static_cast<int64_t>(t) * gh2 * gw2;
        const int64_t unit =
            t_units + (P.order ? static_cast<int64_t>(bw) * gh2 + bh : static_cast<int64_t>(bh) * gw2 + bw);
        const int64_t row = D.row0 + 4 * unit + (mh * 2 + mw);
        const int slot0 = video ? 256 * tt : 0;
        const float2 ly2 = f2(ly, ly), nly2 = f2(-ly, -ly);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            float2 v01 = f2(va[c].x, va[c].y), v23 = f2(va[c].z, va[c].w);
            if (!yident) {
                v01 = fma2(ly2, f2(vb[c].x, vb[c].y), fma2(nly2, v01, v01));
                v23 = fma2(ly2, f2(vb[c].z, vb[c].w), fma2(nly2, v23, v23));
            }
            // an image fills both temporal slots with its one frame; a video half fills slot tt
            store_quad<kBF16>(P, row, c, col, slot0, !video, v01, v23);
        }
        // the merge unit's table entries (once per unit: a video's tt = 0 half): the same entries
        // as write_unit_tables, written inline here because calling that helper from this loop
        // made the bf16 image launch about 1.4% slower
        if (tid < 3 && (!video || tt == 0)) {
            const int64_t src_unit = t_units + static_cast<int64_t>(bh) * gw2 + bw;  // merge order
            const int64_t dst_unit = t_units + static_cast<int64_t>(bw) * gh2 + bh;  // column order
            if (tid == 0 && P.perm != nullptr) {
                const int32_t s0 = static_cast<int32_t>(D.row0 + 4 * src_unit);
                if (MIMO_CHECK(D.row0 + 4 * dst_unit >= 0 && D.row0 + 4 * dst_unit + 4 <= P.chk_table_rows,
                               kChkTableStore))
                    __stcs(reinterpret_cast<int4 *>(P.perm + D.row0 + 4 * dst_unit),
                           make_int4(s0, s0 + 1, s0 + 2, s0 + 3));
            } else if (tid == 1 && P.pos != nullptr) {
                const int32_t h = 2 * bh, w = 2 * bw;
                int4 *d = reinterpret_cast<int4 *>(P.pos + 2 * (D.row0 + 4 * unit));
                if (MIMO_CHECK(D.row0 + 4 * unit >= P.chk_row_lo && D.row0 + 4 * unit + 4 <= P.chk_row_hi,
                               kChkTableStore)) {
                    __stcs(d, make_int4(h, w, h, w + 1));
                    __stcs(d + 1, make_int4(h + 1, w, h + 1, w + 1));
                }
            } else if (tid == 2 && P.win != nullptr) {
                const int64_t u0 = D.row0 / 4;
                if (MIMO_CHECK(u0 + dst_unit >= 0 && 4 * (u0 + dst_unit) + 4 <= P.chk_table_rows, kChkTableStore))
                    P.win[u0 + dst_unit] = static_cast<int32_t>(u0 + src_unit);
            }
        }
        if constexpr (kVideoLaunch) {
            // next half: the other temporal slot of the unit, else one column on, then the next
            // block row, then the next temporal patch (the launch's only item)
            if (tt == 0) {
                tt = 1;
            } else {
                tt = 0;
                if (++bw == gw2) {
                    bw = 0;
                    if (++bh == gh2) {
                        bh = 0;
                        ++t;
                    }
                }
            }
        } else {
            // next block: one column on, then the next block row, then the next image
            if (++bw == gw2) {
                bw = 0;
                if (++bh == gh2) {
                    bh = 0;
                    ++ii;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Warp-staged kernel, for image launches whose images stage both axes' spans
// whole (no gathered axis). Each warp owns the same 4 consecutive output rows
// x 32 columns of every block (the direct kernel's mapping) and stages only the
// source rows those 4 rows need, into its own two-slot slice of shared memory,
// one block ahead with cp.async: nothing waits on more than the warp. A lane
// reads each of its output columns' two taps straight from the staged bytes
// (as the fused RGB step does; RGBA is composited onto white first),
// interpolates along W in its two source rows, then along H, normalises and
// stores as the other kernels do, with the same arithmetic: the outputs are
// bit-identical to the staged kernel's. The taps come from the exact quotient:
// lane l holds the taps of output column l (advanced by 32 columns from block
// to block) and of output row l of the block row, one block ahead, and the
// lanes exchange them with shuffles.
// ---------------------------------------------------------------------------

// Exact tap of output index d along an axis in -> out (den = 2 out), as
// compute_taps forms it: the floor quotient q and remainder r of
// ((2d+1) in - out) / den.
__device__ __forceinline__ void exact_quotient(int64_t d, int32_t in, int32_t out, double inv_den, int32_t &q,
                                               int32_t &r) {
    const int64_t den = 2 * static_cast<int64_t>(out);
    const int64_t num = (2 * d + 1) * in - out;
    int64_t qq = static_cast<int64_t>(floor(static_cast<double>(num) * inv_den));
    int64_t rr = num - qq * den;
    while (rr < 0) {
        --qq;
        rr += den;
    }
    while (rr >= den) {
        ++qq;
        rr -= den;
    }
    q = static_cast<int32_t>(qq);
    r = static_cast<int32_t>(rr);
}

// First tap and weight of the second from (q, r): clamped at 0 from below.
__device__ __forceinline__ void tap_of(int32_t q, int32_t r, float inv_den_f, int32_t &i0, float &lam) {
    const bool clamp = q < 0;
    i0 = clamp ? 0 : q;
    const float rf = (r < (1 << 23)) ? __uint_as_float(0x4B000000u | static_cast<uint32_t>(r)) - kTwo23
                                     : static_cast<float>(r);
    lam = clamp ? 0.0f : rf * inv_den_f;
}

// One block as a warp sees it: its position, the lane's column and row taps
// (lane l: output column l, output row l of the block) and where the warp's
// staged rows start.
struct WarpBlock {
    int ii, bh, bw;
    int32_t ci0, ri0;  // first source column of output column `lane`, first source row of output row `lane`
    float cl, rl;      // their second-tap weights
    int32_t r_lo, c_lo;  // first staged source row (this warp) and first staged source column (the block)
};

template <bool kBF16, class Params>
__global__ void __launch_bounds__(kThreads, 4) warp_kernel(const __grid_constant__ Params P) {
    extern __shared__ float4 smem4[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t B = P.block_start[P.n];
    const int begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * B / gridDim.x);
    const int end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * B / gridDim.x);
    if (begin >= end) return;

    // this thread's place in every block (the direct kernel's mapping)
    const int mh = warp >> 2;
    const int py = ((warp & 3) << 2) | (lane >> 3);
    const int mw = (lane >> 2) & 1;
    const int q = lane & 3;
    const int dy = (mh << 4) | py;
    const int dx0 = (mw << 4) | (q << 2);
    const int col = py * 16 + q * 4;
    const int dy_first = (mh << 4) | ((warp & 3) << 2);  // the warp's first output row in a block
    const int wstride = P.warp_stride;
    const int slot_bytes = P.warp_rows * wstride;
    uint8_t *const wbuf = reinterpret_cast<uint8_t *>(smem4) + static_cast<size_t>(warp) * 2 * slot_bytes;

    // axis constants of the image the cursors are for
    int cur_img = -1;
    int32_t den_x = 1, step_q = 0, step_r = 0, CQ = 1;
    uint32_t cmagic = 1;
    double inv_x = 1.0, inv_y = 1.0;
    float inv_xf = 1.0f, inv_yf = 1.0f;
    // column cursor of output column bw * 32 + lane, row taps of output row bh * 32 + lane
    int32_t cq = 0, cr = 0, rq = 0, rr = 0;
    int row_img = -1, row_bh = -1, col_img = -1, col_bh = -1, col_bw = -2;

    // the taps of block (ii, bh, bw) into wb, and its staging into slot `slot`
    auto prepare = [&](int ii, int bh, int bw, int slot, WarpBlock &wb) {
        const ImageDesc &D = P.img[ii];
        const int32_t H = D.H, W = D.W, Hr = D.Hr, Wr = D.Wr;
        const int C = (D.flags >> kChannelShift) & 0xFF;
        if (ii != cur_img) {
            cur_img = ii;
            den_x = 2 * Wr;
            inv_x = 1.0 / static_cast<double>(den_x);
            inv_xf = static_cast<float>(inv_x);
            inv_y = 1.0 / (2.0 * static_cast<double>(Hr));
            inv_yf = static_cast<float>(inv_y);
            const int64_t step = 2 * static_cast<int64_t>(kBlock) * W;  // numerator change from block to block
            step_q = static_cast<int32_t>(step / den_x);
            step_r = static_cast<int32_t>(step - static_cast<int64_t>(step_q) * den_x);
            // 16-byte chunks covering a staged row segment of the image at any offset
            CQ = (30 + C * (31 * static_cast<int64_t>(W) / Wr + 3)) >> 4;
            cmagic = (65536u + CQ - 1) / CQ;  // job / CQ as (job * cmagic) >> 16, exact for job < 64 * 18
        }
        if (ii == col_img && bh == col_bh && bw == col_bw + 1) {
            cq += step_q;
            cr += step_r;
            if (cr >= den_x) {
                cr -= den_x;
                ++cq;
            }
        } else {
            exact_quotient(static_cast<int64_t>(bw) * kBlock + lane, W, Wr, inv_x, cq, cr);
        }
        col_img = ii;
        col_bh = bh;
        col_bw = bw;
        if (ii != row_img || bh != row_bh) {
            exact_quotient(static_cast<int64_t>(bh) * kBlock + lane, H, Hr, inv_y, rq, rr);
            row_img = ii;
            row_bh = bh;
        }
        wb.ii = ii;
        wb.bh = bh;
        wb.bw = bw;
        tap_of(cq, cr, inv_xf, wb.ci0, wb.cl);
        tap_of(rq, rr, inv_yf, wb.ri0, wb.rl);
        // the warp's source rows and the block's source columns
        const int32_t r_lo = __shfl_sync(0xffffffffu, wb.ri0, dy_first);
        const int32_t r_hi = min(__shfl_sync(0xffffffffu, wb.ri0, dy_first + 3) + 1, H - 1);
        const int32_t c_lo = __shfl_sync(0xffffffffu, wb.ci0, 0);
        const int32_t c_hi = min(__shfl_sync(0xffffffffu, wb.ci0, 31) + 1, W - 1);
        wb.r_lo = r_lo;
        wb.c_lo = c_lo;
        const int nr = r_hi - r_lo + 1;
        const int L = C * (c_hi - c_lo + 1);
        const uint8_t *img = P.src + D.src_off;
        uint8_t *dst = wbuf + slot * slot_bytes;
        for (int job = lane; job < nr * CQ; job += 32) {
            const int j = static_cast<int>((static_cast<uint32_t>(job) * cmagic) >> 16);
            const int c = job - j * CQ;
            const int64_t rs = (static_cast<int64_t>(r_lo + j) * W + c_lo) * C;
            const int64_t cs = (rs & ~int64_t(15)) + 16 * c;
            if (cs < rs + L) {
                const int64_t left = D.limit - cs;
                const int nb = left < 16 ? static_cast<int>(left) : 16;
                if (MIMO_CHECK(cs >= 0 && nb > 0 && cs + nb <= D.limit, kChkSrcCopy) &&
                    MIMO_CHECK(j < P.warp_rows && 16 * c + 16 <= wstride, kChkSmem))
                    cp_async16(dst + j * wstride + 16 * c, img + cs, nb);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    // position of the first block; later blocks advance one column, then one block row, then one image
    int ii = find_image(P, begin);
    int bh, bw;
    {
        const ImageDesc &D = P.img[ii];
        const int g = D.Wr / kBlock;
        const int local = begin - P.block_start[ii] + (ii == 0 ? P.unit0 : 0);
        bh = local / g;
        bw = local - bh * g;
    }
    WarpBlock cur, nxt;
    prepare(ii, bh, bw, 0, cur);
    const float2 m23 = f2(-kTwo23, -kTwo23), neg1 = f2(-1.0f, -1.0f);
    for (int blk = begin; blk < end; ++blk) {
        const int slot = (blk - begin) & 1;
        const bool more = blk + 1 < end;
        if (more) {
            const ImageDesc &D = P.img[ii];
            if (++bw == D.Wr / kBlock) {
                bw = 0;
                if (++bh == D.Hr / kBlock) {
                    bh = 0;
                    ++ii;
                }
            }
            prepare(ii, bh, bw, slot ^ 1, nxt);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();  // every lane's copies of this block have landed

        const ImageDesc &D = P.img[cur.ii];
        const int32_t H = D.H, W = D.W, Hr = D.Hr, Wr = D.Wr;
        const int C = (D.flags >> kChannelShift) & 0xFF;
        const uint8_t *base = wbuf + slot * slot_bytes;
        // this lane's output row and columns
        const int32_t sy0 = __shfl_sync(0xffffffffu, cur.ri0, dy);
        const float ly = __shfl_sync(0xffffffffu, cur.rl, dy);
        const int32_t sy1 = min(sy0 + 1, H - 1);
        int32_t sx[4];
        float lx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            sx[i] = __shfl_sync(0xffffffffu, cur.ci0, dx0 + i);
            lx[i] = __shfl_sync(0xffffffffu, cur.cl, dx0 + i);
        }
        const float2 l01 = f2(lx[0], lx[1]), l23 = f2(lx[2], lx[3]);
        // the quad's values of one staged source row, interpolated along W: h[c] = columns (0,1), (2,3)
        float2 h[2][3][2];
#pragma unroll
        for (int rsel = 0; rsel < 2; ++rsel) {
            const int32_t sy = rsel ? sy1 : sy0;
            const int j = sy - cur.r_lo;
            // byte offset of source column c_lo in the staged row (its 16-byte misalignment)
            const uint32_t mis = ((static_cast<uint32_t>(sy) * static_cast<uint32_t>(W) + static_cast<uint32_t>(cur.c_lo)) *
                                  static_cast<uint32_t>(C)) & 15u;
            const uint8_t *row = base + j * wstride;
            uint32_t a[4], b[4];
            bool ok = MIMO_CHECK(j >= 0 && j < P.warp_rows, kChkSmem);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool next = sx[i] + 1 < W;  // the second tap is the next pixel, or the pixel itself at the edge
                const uint32_t o = mis + static_cast<uint32_t>(C * (sx[i] - cur.c_lo));
                // RGBA reads two aligned words from o, RGB three from o rounded down to a word
                ok = ok && MIMO_CHECK(sx[i] >= cur.c_lo && (C == 4 ? o + 8u : (o & ~3u) + 12u) <= static_cast<uint32_t>(wstride),
                                      kChkSmem);
                if (C == 4) {
                    const uint32_t *w = reinterpret_cast<const uint32_t *>(row + o);
                    a[i] = ok ? w[0] : 0u;
                    b[i] = ok ? (next ? w[1] : a[i]) : 0u;
                } else if (ok) {
                    rgb_pair(row, o, next, a[i], b[i]);
                } else {
                    a[i] = b[i] = 0u;
                }
            }
            if (C == 4) {
                // composite both taps onto white (as the conversion does), then fma(lx, b - a, a)
                const float2 Aa01 = add2(f2(byte_bits<3>(a[0]), byte_bits<3>(a[1])), m23);
                const float2 Aa23 = add2(f2(byte_bits<3>(a[2]), byte_bits<3>(a[3])), m23);
                const float2 Ab01 = add2(f2(byte_bits<3>(b[0]), byte_bits<3>(b[1])), m23);
                const float2 Ab23 = add2(f2(byte_bits<3>(b[2]), byte_bits<3>(b[3])), m23);
                const float2 wa01 = fma2(Aa01, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
                const float2 wa23 = fma2(Aa23, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
                const float2 wb01 = fma2(Ab01, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
                const float2 wb23 = fma2(Ab23, f2(-255.0f, -255.0f), f2(65025.0f, 65025.0f));
#define MIMO_WARP_RGBA(c)                                                                                       \
    {                                                                                                           \
        const float2 A01 = on_white2(add2(f2(byte_bits<c>(a[0]), byte_bits<c>(a[1])), m23), Aa01, wa01);        \
        const float2 A23 = on_white2(add2(f2(byte_bits<c>(a[2]), byte_bits<c>(a[3])), m23), Aa23, wa23);        \
        const float2 B01 = on_white2(add2(f2(byte_bits<c>(b[0]), byte_bits<c>(b[1])), m23), Ab01, wb01);        \
        const float2 B23 = on_white2(add2(f2(byte_bits<c>(b[2]), byte_bits<c>(b[3])), m23), Ab23, wb23);        \
        h[rsel][c][0] = fma2(l01, fma2(A01, neg1, B01), A01);                                                   \
        h[rsel][c][1] = fma2(l23, fma2(A23, neg1, B23), A23);                                                   \
    }
                MIMO_WARP_RGBA(0)
                MIMO_WARP_RGBA(1)
                MIMO_WARP_RGBA(2)
#undef MIMO_WARP_RGBA
            } else {
#define MIMO_WARP_RGB(c)                                                                                        \
    {                                                                                                           \
        const float2 A01 = f2(byte_bits<c>(a[0]), byte_bits<c>(a[1]));                                          \
        const float2 A23 = f2(byte_bits<c>(a[2]), byte_bits<c>(a[3]));                                          \
        h[rsel][c][0] = fma2(l01, fma2(A01, neg1, f2(byte_bits<c>(b[0]), byte_bits<c>(b[1]))), add2(A01, m23)); \
        h[rsel][c][1] = fma2(l23, fma2(A23, neg1, f2(byte_bits<c>(b[2]), byte_bits<c>(b[3]))), add2(A23, m23)); \
    }
                MIMO_WARP_RGB(0)
                MIMO_WARP_RGB(1)
                MIMO_WARP_RGB(2)
#undef MIMO_WARP_RGB
            }
        }
        __syncwarp();  // the slot is read: the next block's copies may reuse it

        // merge order lists units by (block row, block col), column order by (block col, block row)
        const int gw2 = Wr / kBlock, gh2 = Hr / kBlock;
        const int64_t unit = P.order ? static_cast<int64_t>(cur.bw) * gh2 + cur.bh : static_cast<int64_t>(cur.bh) * gw2 + cur.bw;
        const int64_t orow = D.row0 + 4 * unit + (mh * 2 + mw);
        const float2 ly2 = f2(ly, ly), nly2 = f2(-ly, -ly);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const float2 v01 = fma2(ly2, h[1][c][0], fma2(nly2, h[0][c][0], h[0][c][0]));
            const float2 v23 = fma2(ly2, h[1][c][1], fma2(nly2, h[0][c][1], h[0][c][1]));
            store_quad<kBF16>(P, orow, c, col, 0, true, v01, v23);
        }
        if (tid < 3) write_unit_tables(P, tid, D.row0, 0, cur.bh, cur.bw, gh2, gw2, D.row0 + 4 * unit);
        cur = nxt;
    }
}

// Launch setup that depends only on the device and the shared-memory size,
// kept per host thread so that small batches do not pay the driver queries on
// every call.
struct LaunchSetup {
    int dev = -1, sms = 0;
    size_t attr_smem = 0;        // largest dynamic size opted in so far on this device
    size_t occ_smem = ~size_t(0);  // shared-memory size the resident count below is for
    int per_sm = 0;
};

template <bool kBF16, bool kFused, class Params>
int launch_typed(const Params &lp, int64_t blocks, size_t smem_bytes, cudaStream_t stream) {
    auto kern = preprocess_kernel<kBF16, kFused, Params>;
    static thread_local LaunchSetup setup;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ECUDA;
    if (dev != setup.dev) {
        setup = LaunchSetup();
        if (cudaDeviceGetAttribute(&setup.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MIMO_ECUDA;
        setup.dev = dev;
    }
    // the opt-in covers dynamic + static shared memory above the 48 KB default
    if (smem_bytes > setup.attr_smem) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes)) !=
            cudaSuccess)
            return MIMO_ECUDA;
        setup.attr_smem = smem_bytes;
    }
    // persistent grid: as many CTAs as can be resident at once
    if (smem_bytes != setup.occ_smem) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem_bytes) != cudaSuccess ||
            per_sm <= 0)
            return MIMO_ECUDA;
        setup.per_sm = per_sm;
        setup.occ_smem = smem_bytes;
    }
    const int sms = setup.sms, per_sm = setup.per_sm;
    const int64_t grid = std::min<int64_t>(blocks, static_cast<int64_t>(sms) * per_sm);
    kern<<<static_cast<unsigned>(grid), kThreads, smem_bytes, stream>>>(lp);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

template <bool kBF16, bool kVideoLaunch, class Params>
int launch_direct(const Params &lp, int64_t blocks, cudaStream_t stream) {
    auto kern = direct_kernel<kBF16, kVideoLaunch, Params>;
    static thread_local LaunchSetup setup;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ECUDA;
    if (dev != setup.dev) {
        setup = LaunchSetup();
        int per_sm = 0;
        if (cudaDeviceGetAttribute(&setup.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess || per_sm <= 0)
            return MIMO_ECUDA;
        setup.per_sm = per_sm;
        setup.dev = dev;
    }
    // persistent grid, as the staged kernel's
    const int64_t grid = std::min<int64_t>(blocks, static_cast<int64_t>(setup.sms) * setup.per_sm);
    kern<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(lp);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

template <bool kBF16, class Params>
int launch_warp(const Params &lp, int64_t blocks, cudaStream_t stream) {
    auto kern = warp_kernel<kBF16, Params>;
    static thread_local LaunchSetup setup;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MIMO_ECUDA;
    if (dev != setup.dev) {
        setup = LaunchSetup();
        if (cudaDeviceGetAttribute(&setup.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MIMO_ECUDA;
        setup.dev = dev;
    }
    // 8 warps x 2 slots x staged rows x row stride
    const size_t smem_bytes = static_cast<size_t>(kThreads / 32) * 2u * static_cast<size_t>(lp.warp_rows) *
                              static_cast<size_t>(lp.warp_stride);
    if (smem_bytes > setup.attr_smem) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes)) !=
            cudaSuccess)
            return MIMO_ECUDA;
        setup.attr_smem = smem_bytes;
    }
    if (smem_bytes != setup.occ_smem) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem_bytes) != cudaSuccess ||
            per_sm <= 0)
            return MIMO_ECUDA;
        setup.per_sm = per_sm;
        setup.occ_smem = smem_bytes;
    }
    const int64_t grid = std::min<int64_t>(blocks, static_cast<int64_t>(setup.sms) * setup.per_sm);
    kern<<<static_cast<unsigned>(grid), kThreads, smem_bytes, stream>>>(lp);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

// The kernels for one parameter block type, chosen as measured:
//  - the warp-staged kernel for image launches that shrink every image's
//    height by 1.25 or more (and gather no axis): it recomputes both taps of
//    each output pixel, a cost fixed per output, while the staged kernel's
//    conversion and horizontal pass grow with the staged source rows
//    (32 H / Hr + 2 per block); near H = Hr the staged kernel is faster;
//  - the direct kernel when every width is kept, unless fp32 rows of images
//    are written for resized heights (there the staged kernel's burst reads
//    keep the write stream faster). A video half writes one temporal slot,
//    half the stores per staged block, so a video takes the direct kernel in
//    fp32 as well;
//  - the staged kernel otherwise.
template <class Params>
int launch_kernels(const Params &lp, int64_t blocks, int out_dtype, size_t smem_bytes, cudaStream_t s) {
    bool widths_kept = true, heights_kept = true, video = false, fused = false, gather = false, shrunk = true;
    for (int i = 0; i < lp.n; ++i) {
        const int32_t f = lp.img[i].flags;
        gather = gather || (f & (kGatherRows | kGatherCols)) != 0;
        shrunk = shrunk && 4 * static_cast<int64_t>(lp.img[i].H) >= 5 * static_cast<int64_t>(lp.img[i].Hr);
        widths_kept = widths_kept && (f & kIdentityCols) != 0;
        heights_kept = heights_kept && (f & kIdentityRows) != 0;
        video = video || (f & kVideo) != 0;
        // an RGB image with a resized, contiguously staged width takes the fused conversion step
        fused = fused || (((f >> kChannelShift) & 0xFF) == 3 && (f & (kIdentityCols | kGatherCols)) == 0);
    }
    if (!video && !gather && shrunk && lp.warp_rows > 0)
        return out_dtype == MIMO_BF16 ? launch_warp<true>(lp, blocks, s) : launch_warp<false>(lp, blocks, s);
    // a video launch carries exactly one clip
    if (widths_kept && (out_dtype == MIMO_BF16 || heights_kept || video) && (!video || lp.n == 1)) {
        if (video)
            return out_dtype == MIMO_BF16 ? launch_direct<true, true>(lp, blocks, s)
                                          : launch_direct<false, true>(lp, blocks, s);
        return out_dtype == MIMO_BF16 ? launch_direct<true, false>(lp, blocks, s)
                                      : launch_direct<false, false>(lp, blocks, s);
    }
    // the staged kernel with the fused RGB step only where a launch needs it: it costs registers
    // (and measurably some time) in launches that never take it
    if (fused)
        return out_dtype == MIMO_BF16 ? launch_typed<true, true>(lp, blocks, smem_bytes, s)
                                      : launch_typed<false, true>(lp, blocks, smem_bytes, s);
    return out_dtype == MIMO_BF16 ? launch_typed<true, false>(lp, blocks, smem_bytes, s)
                                  : launch_typed<false, false>(lp, blocks, smem_bytes, s);
}

}  // namespace

namespace {
// Drops 128-byte lines from L2 without writing them back to HBM. The chained
// pixels-to-embeddings call runs it over a scratch half once the GEMM has read
// it: those rows are dead, and writing them back would cost HBM bandwidth.
__global__ void discard_l2_kernel(uint8_t *p, int64_t lines) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < lines;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        asm volatile("discard.global.L2 [%0], 128;" ::"l"(p + 128 * i) : "memory");
}
}  // namespace

int launch_discard_l2(void *p, int64_t bytes, void *stream) {
    if ((reinterpret_cast<uintptr_t>(p) & 127u) != 0) return MIMO_EALIGN;
    const int64_t lines = bytes / 128;
    if (lines <= 0) return MIMO_OK;
    const int64_t blocks = std::min<int64_t>((lines + 255) / 256, 148 * 8);
    discard_l2_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint8_t *>(p), lines);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

int bounds_check_status(int64_t *violations, int32_t *first_kind) {
#if defined(MIMO_BOUNDS_CHECK)
    unsigned long long v = 0;
    int k = 0;
    if (cudaMemcpyFromSymbol(&v, g_bounds_violations, sizeof(v)) != cudaSuccess ||
        cudaMemcpyFromSymbol(&k, g_bounds_first_kind, sizeof(k)) != cudaSuccess)
        return MIMO_ECUDA;
    const unsigned long long zero = 0;
    const int zk = 0;
    if (cudaMemcpyToSymbol(g_bounds_violations, &zero, sizeof(zero)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_bounds_first_kind, &zk, sizeof(zk)) != cudaSuccess)
        return MIMO_ECUDA;
    *violations = static_cast<int64_t>(v);
    *first_kind = k;
    return MIMO_OK;
#else
    (void)violations;
    (void)first_kind;
    return MIMO_EUNSUPPORTED;
#endif
}

int launch_preprocess(const LaunchParams &lp, int64_t blocks, int out_dtype, size_t smem_bytes, void *stream) {
    if (blocks <= 0) return MIMO_OK;
    if (blocks > static_cast<int64_t>(INT32_MAX)) return MIMO_EOVERFLOW;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (lp.n <= kSmallLaunch) {
        // a few images: copy into the small parameter block (the launch then costs about half)
        static thread_local SmallLaunchParams sp;
        std::memcpy(&sp, &lp, offsetof(LaunchParams, block_start));
        std::memcpy(sp.block_start, lp.block_start, sizeof(int32_t) * (lp.n + 1));
        std::memcpy(sp.img, lp.img, sizeof(ImageDesc) * lp.n);
        return launch_kernels(sp, blocks, out_dtype, smem_bytes, s);
    }
    return launch_kernels(lp, blocks, out_dtype, smem_bytes, s);
}

}  // namespace mimo
