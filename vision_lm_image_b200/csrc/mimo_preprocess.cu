// mimo_preprocess.cu -- the fused MiMo-V2 pixel path for sm_100a.
//
// One CTA owns one 32x32 merge block of one resized image (4 output rows of
// 1536 values) and does every step of the path for it:
//   0. exact bilinear taps of its 32 output rows (warp 0) and 32 output
//      columns (warp 1) under align_corners=False (NeMo Automodel
//      "mimo_v2_flash.processing", class MimoV2ImageProcessor: F.interpolate
//      bilinear; docs.rs "cortiq_engine::mimo_vision", resize_bilinear);
//   1. stages the source samples those taps touch into shared memory as
//      planar fp32 on the 0..255 scale, compositing RGBA onto white on the
//      way in (function _to_rgb); each lane moves 4 source pixels with
//      aligned 32-bit loads and 16-byte shared stores;
//   2. interpolates along W for every staged row (skipped when the width is
//      not resized), then along H with packed f32x2 arithmetic, applies
//      (x - 255*mean)/(255*std) folded to x*k + b (module docstring), and
//      writes each 16-pixel row segment twice, once per temporal frame, laid
//      out (c, tt, py, px) in merge-block row order (cortiq page, conventions);
//   3. writes the column-order permutation entries of its merge unit
//      (cortiq page, column_permutation).
// The kernel has no inter-CTA communication, no atomics and no waits; every
// output element has exactly one writer.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mimo.h"
#include "mimo_internal.h"

namespace mimo {
namespace {

constexpr float kTwo23 = 8388608.0f;

// Byte k of w as an exact float: PRMT builds the bit pattern 0x4B0000bb
// (= 2^23 + b) and one subtraction removes 2^23.
template <int k>
__device__ __forceinline__ float byte_f(uint32_t w) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u + k)) - kTwo23;
}

// Composite one RGBA channel value onto white: nearest integer of
// (c*a + 255*(255-a)) / 255, as an exact float. 255 is odd, so there are no
// ties, and floor((t + 127.5) / 255) equals floor((t + 127) / 255).
__device__ __forceinline__ float on_white(uint32_t c, uint32_t a, uint32_t white) {
    const uint32_t t = c * a + white;  // white = 255 * (255 - a)
    return __uint_as_float(0x4B000000u | ((t + 127u) / 255u)) - kTwo23;
}

__device__ __forceinline__ uint64_t pack2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
    return f;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// last i with block_start[i] <= blk
__device__ __forceinline__ int find_image(const LaunchParams &P, int blk) {
    int lo = 0, hi = P.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.block_start[mid] <= blk) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// One 32-bit word of the image at word index a (byte 4a), or, for the last
// partial word of an image that ends unaligned at the end of the caller's
// buffer, its bytes below `size` (the rest zero).
__device__ __forceinline__ uint32_t load_word(const uint8_t *img, int64_t a, int64_t readable, int64_t size) {
    if (4 * a + 4 <= readable) return __ldg(reinterpret_cast<const uint32_t *>(img) + a);
    uint32_t w = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b)
        if (4 * a + b < size) w |= static_cast<uint32_t>(__ldg(img + 4 * a + b)) << (8 * b);
    return w;
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads) preprocess_kernel(const __grid_constant__ LaunchParams P) {
    extern __shared__ float4 smem4[];
    float *const tile = reinterpret_cast<float *>(smem4);  // [3][tile_rows][tile_stride] (+ hbuf)
    __shared__ int32_t s_img;
    __shared__ int32_t s_ty[2][kBlock];
    __shared__ int32_t s_tx[2][kBlock];
    __shared__ float s_ly[kBlock];
    __shared__ float s_lx[kBlock];
    __shared__ int32_t s_srow[kMaxTile];
    __shared__ int32_t s_scol[kMaxTile];
    __shared__ int32_t s_span[4];  // first row, rows, first col, cols

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int blk = blockIdx.x;

    // ---- 0. taps: warp 0 -> the block's 32 output rows, warp 1 -> columns
    if (warp < 2) {
        const int ii = find_image(P, blk);
        const ImageDesc &D = P.img[ii];
        const int local = blk - P.block_start[ii];
        const int gw2 = D.Wr / kBlock;
        const int bh = local / gw2;
        const int bw = local - bh * gw2;
        const bool is_col = warp == 1;
        const int64_t in = is_col ? D.W : D.H;
        const int64_t out = is_col ? D.Wr : D.Hr;
        const bool gather = (D.flags & (is_col ? kGatherCols : kGatherRows)) != 0;
        const bool ident = (D.flags & (is_col ? kIdentityCols : kIdentityRows)) != 0;
        const int64_t d = static_cast<int64_t>(is_col ? bw : bh) * kBlock + lane;
        // source coordinate ((2d+1)*in - out) / (2*out): fp64 quotient, exact
        // integer correction
        const int64_t num = (2 * d + 1) * in - out;
        const int64_t den = 2 * out;
        int64_t q = 0, r = 0;
        if (num > 0) {
            q = static_cast<int64_t>(static_cast<double>(num) / static_cast<double>(den));
            r = num - q * den;
            if (r < 0) {
                --q;
                r += den;
            } else if (r >= den) {
                ++q;
                r -= den;
            }
        }
        const int32_t i0 = static_cast<int32_t>(q);
        const int32_t i1 = (q + 1 < in) ? i0 + 1 : static_cast<int32_t>(in - 1);
        const float lam = __fdiv_rn(static_cast<float>(r), static_cast<float>(den));
        const int32_t first = __shfl_sync(0xffffffffu, i0, 0);
        const int32_t last = __shfl_sync(0xffffffffu, i1, 31);
        int32_t j0, j1, count;
        if (gather) {
            j0 = 2 * lane;
            j1 = 2 * lane + 1;
            int32_t *src_idx = is_col ? s_scol : s_srow;
            src_idx[j0] = i0;
            src_idx[j1] = i1;
            count = kMaxTile;
        } else {
            j0 = i0 - first;
            j1 = i1 - first;
            count = ident ? kBlock : last - first + 1;
        }
        if (is_col) {
            s_tx[0][lane] = j0;
            s_tx[1][lane] = j1;
            s_lx[lane] = lam;
        } else {
            s_ty[0][lane] = j0;
            s_ty[1][lane] = j1;
            s_ly[lane] = lam;
        }
        if (lane == 0) {
            s_span[is_col ? 2 : 0] = gather ? 0 : first;
            s_span[is_col ? 3 : 1] = count;
            if (!is_col) s_img = ii;
        }
    }
    __syncthreads();

    const int ii = s_img;
    const ImageDesc &D = P.img[ii];
    const int flags = D.flags;
    const int TS = P.tile_stride;
    const int plane = P.tile_rows * TS;
    const int y_first = s_span[0], nrows = s_span[1];
    const int x_first = s_span[2], ncols = s_span[3];

    // ---- 1. stage source samples as planar fp32, RGBA composited onto white
    {
        const uint8_t *img = P.src + D.src_off;
        const int64_t W = D.W;
        const bool grow = (flags & kGatherRows) != 0;
        if ((flags & kGatherCols) == 0) {
            // a job = 4 consecutive staged pixels of one tile row
            const int Q = (ncols + 3) >> 2;
            const uint32_t qmagic = (65536u + Q - 1) / Q;  // job / Q exact for job < 1024, Q <= 16
            const int jobs = nrows * Q;
            for (int job = tid; job < jobs; job += kThreads) {
                const int j = static_cast<int>((static_cast<uint32_t>(job) * qmagic) >> 16);
                const int px0 = (job - j * Q) * 4;
                const int sy = grow ? s_srow[j] : y_first + j;
                const int64_t pix0 = static_cast<int64_t>(sy) * W + x_first + px0;  // first source pixel
                float4 c0, c1, c2;
                if (D.C == 4) {
                    const int nv = min(4, ncols - px0);
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        w[k] = (k < nv) ? __ldg(reinterpret_cast<const uint32_t *>(img) + pix0 + k) : 0xFF000000u;
                    float o[3][4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t a = w[k] >> 24;
                        const uint32_t white = 255u * (255u - a);
                        o[0][k] = on_white(w[k] & 0xFFu, a, white);
                        o[1][k] = on_white((w[k] >> 8) & 0xFFu, a, white);
                        o[2][k] = on_white((w[k] >> 16) & 0xFFu, a, white);
                    }
                    c0 = make_float4(o[0][0], o[0][1], o[0][2], o[0][3]);
                    c1 = make_float4(o[1][0], o[1][1], o[1][2], o[1][3]);
                    c2 = make_float4(o[2][0], o[2][1], o[2][2], o[2][3]);
                } else {
                    // 12 bytes from byte 3*pix0: up to 4 aligned words, realigned
                    const int64_t b0 = 3 * pix0;
                    const int64_t a0 = b0 >> 2;
                    const int sh = static_cast<int>(b0 & 3) * 8;
                    const int64_t bend = 3 * (pix0 + min(4, ncols - px0));  // end of the bytes needed
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        w[k] = (4 * (a0 + k) < bend) ? load_word(img, a0 + k, D.readable, 3 * (int64_t)D.H * W) : 0u;
                    const uint32_t r0 = __funnelshift_r(w[0], w[1], sh);
                    const uint32_t r1 = __funnelshift_r(w[1], w[2], sh);
                    const uint32_t r2 = __funnelshift_r(w[2], w[3], sh);
                    // bytes: r0 = R0 G0 B0 R1 | r1 = G1 B1 R2 G2 | r2 = B2 R3 G3 B3
                    c0 = make_float4(byte_f<0>(r0), byte_f<3>(r0), byte_f<2>(r1), byte_f<1>(r2));
                    c1 = make_float4(byte_f<1>(r0), byte_f<0>(r1), byte_f<3>(r1), byte_f<2>(r2));
                    c2 = make_float4(byte_f<2>(r0), byte_f<1>(r1), byte_f<0>(r2), byte_f<3>(r2));
                }
                float *t = tile + j * TS + px0;
                *reinterpret_cast<float4 *>(t) = c0;
                *reinterpret_cast<float4 *>(t + plane) = c1;
                *reinterpret_cast<float4 *>(t + 2 * plane) = c2;
            }
        } else {
            // gathered columns: 64 single pixels per tile row
            const int total = nrows * kMaxTile;
            for (int e = tid; e < total; e += kThreads) {
                const int j = e >> 6;
                const int i = e & (kMaxTile - 1);
                const int sy = grow ? s_srow[j] : y_first + j;
                const int64_t pix = static_cast<int64_t>(sy) * W + s_scol[i];
                float r, g, b;
                if (D.C == 4) {
                    const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(img) + pix);
                    const uint32_t a = v >> 24;
                    const uint32_t white = 255u * (255u - a);
                    r = on_white(v & 0xFFu, a, white);
                    g = on_white((v >> 8) & 0xFFu, a, white);
                    b = on_white((v >> 16) & 0xFFu, a, white);
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
    __syncthreads();

    // ---- 2a. horizontal pass (resized widths only): hbuf[c][j][dx]
    const bool hpass = (flags & kIdentityCols) == 0;
    if (hpass) {
        float *hb = tile + P.hbuf;
        const int hplane = P.tile_rows * kBlock;
        const int x0 = s_tx[0][lane], x1 = s_tx[1][lane];
        const float lx = s_lx[lane];
        for (int j = warp; j < nrows; j += kThreads / 32) {
            const float *t = tile + j * TS;
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                const float a = t[c * plane + x0];
                const float b = t[c * plane + x1];
                hb[c * hplane + j * kBlock + lane] = fmaf(lx, b - a, a);
            }
        }
        __syncthreads();
    }

    // ---- 2b. vertical pass + normalisation + both temporal copies
    // warp w covers output rows dy = 4w..4w+3 of the block; a lane covers 4
    // consecutive columns. For fixed mw the 16 lanes write 4 consecutive
    // 16-float segments of one output row: 256 contiguous bytes (fp32).
    {
        const int mh = warp >> 2;
        const int py = ((warp & 3) << 2) | (lane >> 3);
        const int mw = (lane >> 2) & 1;
        const int q = lane & 3;
        const int dy = (mh << 4) | py;
        const int dx0 = (mw << 4) | (q << 2);
        const float *buf = hpass ? tile + P.hbuf : tile;
        const int stride = hpass ? kBlock : TS;
        const int vplane = hpass ? P.tile_rows * kBlock : plane;
        const bool yident = (flags & kIdentityRows) != 0;
        const int r0 = s_ty[0][dy] * stride + dx0;
        const int r1 = s_ty[1][dy] * stride + dx0;
        const float ly = s_ly[dy];
        const uint64_t ly2 = pack2(ly, ly);

        const int local = blk - P.block_start[ii];
        const int gw2 = D.Wr / kBlock;
        const int bh = local / gw2;
        const int bw = local - bh * gw2;
        const int64_t row = D.row0 + 4LL * (static_cast<int64_t>(bh) * gw2 + bw) + (mh * 2 + mw);
        const int col = py * 16 + q * 4;
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const float4 A = *reinterpret_cast<const float4 *>(buf + c * vplane + r0);
            uint64_t v01 = pack2(A.x, A.y), v23 = pack2(A.z, A.w);
            if (!yident) {
                const float4 B = *reinterpret_cast<const float4 *>(buf + c * vplane + r1);
                v01 = fma2(ly2, sub2(pack2(B.x, B.y), v01), v01);
                v23 = fma2(ly2, sub2(pack2(B.z, B.w), v23), v23);
            }
            const uint64_t k2 = pack2(P.k[c], P.k[c]), b2 = pack2(P.b[c], P.b[c]);
            const float2 n01 = unpack2(fma2(v01, k2, b2));
            const float2 n23 = unpack2(fma2(v23, k2, b2));
            if constexpr (!kBF16) {
                float *o = static_cast<float *>(P.out) + row * kRowWidth + c * 512 + col;
                const float4 f4 = make_float4(n01.x, n01.y, n23.x, n23.y);
                __stcs(reinterpret_cast<float4 *>(o), f4);        // tt = 0
                __stcs(reinterpret_cast<float4 *>(o + 256), f4);  // tt = 1
            } else {
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(P.out) + row * kRowWidth + c * 512 + col;
                const __nv_bfloat162 lo2 = __floats2bfloat162_rn(n01.x, n01.y);
                const __nv_bfloat162 hi2 = __floats2bfloat162_rn(n23.x, n23.y);
                uint2 u;
                u.x = *reinterpret_cast<const uint32_t *>(&lo2);
                u.y = *reinterpret_cast<const uint32_t *>(&hi2);
                __stcs(reinterpret_cast<uint2 *>(o), u);
                __stcs(reinterpret_cast<uint2 *>(o + 256), u);
            }
        }

        // ---- 3. column-order permutation: unit (bh, bw) is listed at (bw, bh)
        if (P.perm != nullptr && tid == 0) {
            const int gh2 = D.Hr / kBlock;
            const int64_t src_unit = static_cast<int64_t>(bh) * gw2 + bw;
            const int64_t dst_unit = static_cast<int64_t>(bw) * gh2 + bh;
            const int32_t s0 = static_cast<int32_t>(D.row0 + 4 * src_unit);
            __stcs(reinterpret_cast<int4 *>(P.perm + D.row0 + 4 * dst_unit), make_int4(s0, s0 + 1, s0 + 2, s0 + 3));
        }
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
