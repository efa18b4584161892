// mimo_preprocess.cu -- the fused MiMo-V2 pixel path for sm_100a.
//
// One CTA owns one 32x32 merge block of one resized image (4 output rows of
// 1536 values) and does every step of the path for it:
//   1. exact bilinear taps of its 32 output rows and 32 output columns
//      (align_corners=False; NeMo Automodel "mimo_v2_flash.processing",
//      class MimoV2ImageProcessor: F.interpolate bilinear; docs.rs
//      "cortiq_engine::mimo_vision", resize_bilinear);
//   2. stages the source samples those taps touch into shared memory as
//      planar fp32 on the 0..255 scale, compositing RGBA onto white on the
//      way in (function _to_rgb);
//   3. interpolates along W on the two source rows, then along H, applies
//      (x - 255*mean)/(255*std) folded to x*k + b (module docstring), and
//      writes each 16-pixel row segment twice, once per temporal frame,
//      laid out (c, tt, py, px) in merge-block row order (cortiq page,
//      conventions list);
//   4. writes the column-order permutation entries of its merge unit
//      (cortiq page, column_permutation).
// The kernel has no inter-CTA communication, no atomics and no waits; every
// output element has exactly one writer.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mimo.h"
#include "mimo_internal.h"

namespace mimo {
namespace {

// Exact uint8 -> float: 2^23 + v is representable for v < 2^23, so the
// subtraction returns v exactly (an integer add and an FP add instead of a
// conversion instruction).
__device__ __forceinline__ float byte_to_float(uint32_t v) {
    return __uint_as_float(0x4B000000u | v) - 8388608.0f;
}

// Composite one RGBA channel value onto white: nearest integer of
// (c*a + 255*(255-a)) / 255. 255 is odd, so there are no ties, and
// floor((t + 127.5) / 255) equals floor((t + 127) / 255) for integer t.
__device__ __forceinline__ uint32_t on_white(uint32_t c, uint32_t a) {
    const uint32_t t = c * a + 255u * (255u - a);
    return (t + 127u) / 255u;
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads) preprocess_kernel(const __grid_constant__ LaunchParams P) {
    extern __shared__ float tile[];  // [3][tile_rows][tile_stride]
    __shared__ int32_t s_src_row[kMaxTile];
    __shared__ int32_t s_src_col[kMaxTile];
    __shared__ int32_t s_ty[2][kBlock];
    __shared__ int32_t s_tx[2][kBlock];
    __shared__ float s_ly[kBlock];
    __shared__ float s_lx[kBlock];
    __shared__ int32_t s_span[4];  // first row, rows, first col, cols

    const int tid = threadIdx.x;
    const int blk = blockIdx.x;

    // the image this block belongs to: last i with block_start[i] <= blk
    int lo = 0, hi = P.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.block_start[mid] <= blk) lo = mid;
        else hi = mid - 1;
    }
    const ImageDesc D = P.img[lo];
    const int local = blk - P.block_start[lo];
    const int gw2 = D.Wr / kBlock;
    const int gh2 = D.Hr / kBlock;
    const int bh = local / gw2;
    const int bw = local - bh * gw2;

    // ---- 1. taps: threads 0..31 -> output rows, 32..63 -> output columns
    if (tid < 2 * kBlock) {
        const bool is_col = tid >= kBlock;
        const int d = tid & (kBlock - 1);
        const int64_t in = is_col ? D.W : D.H;
        const int64_t out = is_col ? D.Wr : D.Hr;
        const int64_t base = static_cast<int64_t>(is_col ? bw : bh) * kBlock;
        const bool gather = (D.flags & (is_col ? kGatherCols : kGatherRows)) != 0;
        const Taps t = axis_taps(base + d, in, out);
        const float lam = static_cast<float>(static_cast<double>(t.rem) / static_cast<double>(t.den));
        int32_t first = 0, j0, j1;
        if (gather) {
            j0 = 2 * d;
            j1 = 2 * d + 1;
            int32_t *src_idx = is_col ? s_src_col : s_src_row;
            src_idx[j0] = static_cast<int32_t>(t.i0);
            src_idx[j1] = static_cast<int32_t>(t.i1);
        } else {
            first = static_cast<int32_t>(axis_taps(base, in, out).i0);
            j0 = static_cast<int32_t>(t.i0) - first;
            j1 = static_cast<int32_t>(t.i1) - first;
        }
        if (is_col) {
            s_tx[0][d] = j0;
            s_tx[1][d] = j1;
            s_lx[d] = lam;
        } else {
            s_ty[0][d] = j0;
            s_ty[1][d] = j1;
            s_ly[d] = lam;
        }
        if (d == kBlock - 1) {
            s_span[is_col ? 2 : 0] = first;
            s_span[is_col ? 3 : 1] = gather ? kMaxTile : j1 + 1;
        }
    }
    __syncthreads();

    // ---- 2. stage the source samples as planar fp32, RGBA onto white
    const int TS = P.tile_stride;
    const int plane = P.tile_rows * TS;
    {
        const int y_first = s_span[0], nrows = s_span[1];
        const int x_first = s_span[2], ncols = s_span[3];
        const bool grow = (D.flags & kGatherRows) != 0;
        const bool gcol = (D.flags & kGatherCols) != 0;
        const uint8_t *img = P.src + D.src_off;
        const int total = nrows * ncols;
        const float inv_ncols = 1.0f / static_cast<float>(ncols);
        for (int idx = tid; idx < total; idx += kThreads) {
            // idx < 64*64: (idx + 0.5)/ncols is at least 0.5/64 away from an
            // integer, far above the fp32 error, so j is exact
            const int j = static_cast<int>((static_cast<float>(idx) + 0.5f) * inv_ncols);
            const int i = idx - j * ncols;
            const int sy = grow ? s_src_row[j] : y_first + j;
            const int sx = gcol ? s_src_col[i] : x_first + i;
            const int64_t pix = static_cast<int64_t>(sy) * D.W + sx;
            float r, g, b;
            if (D.C == 4) {
                const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(img) + pix);
                const uint32_t a = v >> 24;
                r = byte_to_float(on_white(v & 0xFFu, a));
                g = byte_to_float(on_white((v >> 8) & 0xFFu, a));
                b = byte_to_float(on_white((v >> 16) & 0xFFu, a));
            } else {
                const uint8_t *px = img + pix * 3;
                r = byte_to_float(__ldg(px));
                g = byte_to_float(__ldg(px + 1));
                b = byte_to_float(__ldg(px + 2));
            }
            float *t = tile + j * TS + i;
            t[0] = r;
            t[plane] = g;
            t[2 * plane] = b;
        }
    }
    __syncthreads();

    // ---- 3. interpolate + normalise + store both temporal copies
    // warp w covers output rows dy = 4w..4w+3 of the block; a lane covers 4
    // consecutive columns. For fixed mw the 16 lanes write 4 consecutive
    // 16-float segments of one output row: 256 contiguous bytes (fp32).
    const int warp = tid >> 5, lane = tid & 31;
    const int mh = warp >> 2;
    const int py = ((warp & 3) << 2) | (lane >> 3);
    const int mw = (lane >> 2) & 1;
    const int q = lane & 3;
    const int dy = (mh << 4) | py;
    const int dx0 = (mw << 4) | (q << 2);
    const int ry0 = s_ty[0][dy] * TS;
    const int ry1 = s_ty[1][dy] * TS;
    const float ly = s_ly[dy];
    int cx0[4], cx1[4];
    float lx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        cx0[k] = s_tx[0][dx0 + k];
        cx1[k] = s_tx[1][dx0 + k];
        lx[k] = s_lx[dx0 + k];
    }
    const int64_t row = D.row0 + 4LL * (static_cast<int64_t>(bh) * gw2 + bw) + (mh * 2 + mw);
    const int col = py * 16 + q * 4;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        const float *t0 = tile + c * plane + ry0;
        const float *t1 = tile + c * plane + ry1;
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float a = t0[cx0[k]], b = t0[cx1[k]];
            const float e = t1[cx0[k]], f = t1[cx1[k]];
            const float top = fmaf(lx[k], b - a, a);
            const float bot = fmaf(lx[k], f - e, e);
            const float s = fmaf(ly, bot - top, top);
            v[k] = fmaf(s, P.k[c], P.b[c]);
        }
        if constexpr (!kBF16) {
            float *o = static_cast<float *>(P.out) + row * kRowWidth + c * 512 + col;
            const float4 f4 = make_float4(v[0], v[1], v[2], v[3]);
            __stcs(reinterpret_cast<float4 *>(o), f4);        // tt = 0
            __stcs(reinterpret_cast<float4 *>(o + 256), f4);  // tt = 1
        } else {
            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(P.out) + row * kRowWidth + c * 512 + col;
            const __nv_bfloat162 lo2 = __floats2bfloat162_rn(v[0], v[1]);
            const __nv_bfloat162 hi2 = __floats2bfloat162_rn(v[2], v[3]);
            uint2 u;
            u.x = *reinterpret_cast<const uint32_t *>(&lo2);
            u.y = *reinterpret_cast<const uint32_t *>(&hi2);
            __stcs(reinterpret_cast<uint2 *>(o), u);
            __stcs(reinterpret_cast<uint2 *>(o + 256), u);
        }
    }

    // ---- 4. column-order permutation: unit (bh, bw) is listed at (bw, bh)
    if (P.perm != nullptr && tid == 0) {
        const int64_t src_unit = static_cast<int64_t>(bh) * gw2 + bw;
        const int64_t dst_unit = static_cast<int64_t>(bw) * gh2 + bh;
        const int32_t s0 = static_cast<int32_t>(D.row0 + 4 * src_unit);
        __stcs(reinterpret_cast<int4 *>(P.perm + D.row0 + 4 * dst_unit), make_int4(s0, s0 + 1, s0 + 2, s0 + 3));
    }
}

template <bool kBF16>
int launch_typed(const LaunchParams &lp, int64_t blocks, size_t smem_bytes, cudaStream_t stream) {
    auto kern = preprocess_kernel<kBF16>;
    if (smem_bytes > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes)) !=
            cudaSuccess)
            return MIMO_ECUDA;
    }
    kern<<<static_cast<unsigned>(blocks), kThreads, smem_bytes, stream>>>(lp);
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

}  // namespace

int launch_preprocess(const LaunchParams &lp, int64_t blocks, int out_dtype, size_t smem_bytes, void *stream) {
    if (blocks <= 0) return MIMO_OK;
    if (blocks > static_cast<int64_t>(INT32_MAX)) return MIMO_EOVERFLOW;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return out_dtype == MIMO_BF16 ? launch_typed<true>(lp, blocks, smem_bytes, s)
                                  : launch_typed<false>(lp, blocks, smem_bytes, s);
}

}  // namespace mimo
