// mimo_patch_embed.cu -- the vision tower's patch embedding on the 5th-gen
// tensor cores (NeMo Automodel "mimo_v2_flash.vision", MiMoVisionPatchEmbed:
// flattened spatiotemporal patches to vision tokens). The Conv3d with kernel =
// stride = (2, 16, 16) is a dense contraction of each 1536-value patch row
// with a [embed_dim, 1536] weight laid out (c, tt, py, px), the same order as
// the rows:
//
//   C[m, n] = sum_k A[m, k] * B[n, k] (+ bias[n]),  A = patch rows (bf16),
//   B = weight (bf16), accumulated in fp32, C in bf16 or fp32.
//
// Persistent kernel on CTA pairs (clusters of two SMs), walking the 256 x 256
// tiles of C in m-major order (the embed_dim / 256 tiles that share rows run
// side by side, so each row block is read from HBM once). Each CTA of a pair
// holds half of A (128 rows) and half of B (128 of the 256 weight rows) per
// 128-wide K block, as two 64-wide halves in the 128-byte swizzle; warp 0 of
// each CTA streams its A with TMA and warp 6 its B, into a 3-stage ring, and
// all of it signals the even CTA's barrier. One lane of the even CTA issues
// tcgen05.mma.cta_group::2 (M256 N256 K16: the tensor cores of both SMs, each
// reading its own half of A and both halves of B), eight per stage, and frees
// each stage in both CTAs with a multicast tcgen05.commit. A stage of 128 K
// (1024 tensor-core cycles per SM) rather than 64 is what lets one thread keep
// the tensor pipe fed: each barrier wait, copy issue and commit costs that
// thread a few hundred cycles, and one tcgen05.mma about 80. Warps 2-5 of
// each CTA drain their 128 accumulator rows with tcgen05.ld, add the bias,
// convert and store. TMEM holds two accumulators (2 x 256 columns) per CTA, so
// the epilogue of one tile runs under the MMAs of the next. Splitting the tile
// across the pair halves the weight bytes each SM stages per MMA.
// Every wait on an mbarrier is bounded: on expiry the kernel records an error
// code in *err, every role stops issuing work, the producer waits (bounded) for
// the copies it started, the MMA lane for the MMAs it issued, and the TMEM is
// freed before exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "mimo.h"
#include "mimo_internal.h"

namespace mimo {
namespace {

constexpr int kPairM = 256;                // rows of C per tile (128 per CTA of the pair)
constexpr int kBM = 128;                    // rows of A per CTA
constexpr int kBN = 256;                    // columns of C per tile
constexpr int kBNHalf = kBN / 2;            // weight rows per CTA
constexpr int kBK = 128;                    // K per stage
constexpr int kAtomK = 64;                  // kAtomK * 2 B = one 128-byte swizzle row (one TMA box)
constexpr int kStages = 3;
constexpr int kUmmaK = 16;
constexpr int kAAtomBytes = kBM * kAtomK * 2;      // 16 KB: 128 rows of one 64-wide half
constexpr int kBAtomBytes = kBNHalf * kAtomK * 2;  // 16 KB
constexpr int kATileBytes = kBM * kBK * 2;         // 32 KB
constexpr int kBTileBytes = kBNHalf * kBK * 2;     // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kGemmThreads = 224;           // 7 warps: A loader, MMA, 4 epilogue, B loader
constexpr int kAccCols = kBN;               // one fp32 accumulator: 128 lanes x 256 columns per CTA
constexpr int kTmemCols = 2 * kAccCols;     // double-buffered
constexpr int kEpiWarps = 4;
constexpr int kStagePitch = 128 + 16;       // epilogue staging row: one 128-byte output line + pad (no bank conflicts)
constexpr int kEpiStageBytes = 32 * kStagePitch;  // per epilogue warp: 32 rows
constexpr uint16_t kPairMask = 0x3;         // both CTAs of the cluster
constexpr uint32_t kWaitLimit = 1u << 20;   // try_wait rounds before a wait is declared stuck (default)

enum : int { kErrNone = 0, kErrFullWait = 1, kErrEmptyWait = 2, kErrAccumWait = 3, kErrAccumFreeWait = 4,
             kErrDrainWait = 5 };

struct GemmSmem {
    uint64_t full[kStages];   // even CTA: both halves of stage s landed (TMA of both CTAs)
    uint64_t empty[kStages];  // each CTA: the pair's MMAs consumed stage s (multicast commit)
    uint64_t acc_full[2];     // each CTA: accumulator b complete (multicast commit)
    uint64_t acc_free[2];     // even CTA: all 8 epilogue warps of the pair drained accumulator b
    uint64_t drain;           // even CTA: every MMA it issued has completed
    uint32_t tmem_base;
    int32_t failed;           // a role of this CTA gave up waiting: the others stop too
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Arrive on a barrier given by its shared::cluster address (possibly the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// Bounded wait for the phase with the given parity to complete; false if
// `limit` try_wait rounds ran out (the caller records the error and stops).
// Cluster scope: some of the arrivals come from the other CTA of the pair.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t limit) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ bool stopped(const GemmSmem &S) {
    return *reinterpret_cast<const volatile int32_t *>(&S.failed) != 0;
}

__device__ __forceinline__ void fail(GemmSmem &S, int32_t *err, int code) {
    atomicCAS(err, kErrNone, code);
    *reinterpret_cast<volatile int32_t *>(&S.failed) = 1;
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// the barrier at `cluster_bar` (the even CTA's, for both CTAs of the pair).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t cluster_bar, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(x), "r"(y)
        : "memory");
}

// Arrive on the barrier at the same offset in both CTAs once the MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(kPairMask)
        : "memory");
}

__device__ __forceinline__ void umma_commit_local(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor of a K-major tile stored as 128-byte rows
// with the 128-byte swizzle (what TMA writes with CU_TENSOR_MAP_SWIZZLE_128B):
// start address >> 4, leading offset 16 B (unused by this layout), stride
// 1024 B between groups of 8 rows, descriptor version 1, layout 128B swizzle.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 256 (the pair's tile).
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | ((kPairM >> 4) << 24);

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

// 32 fp32 accumulator columns of this lane's row (+ bias) -> 128 or 64 bytes
// of output at byte offset `off` of the lane's staging row.
template <bool kOutBF16>
__device__ __forceinline__ void stage_32(uint8_t *srow, int off, const uint32_t (&v)[32],
                                         const float *__restrict__ bias, int col) {
    float f[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]) + (bias ? __ldg(bias + col + j) : 0.0f);
    if constexpr (kOutBF16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 p0 = __floats2bfloat162_rn(f[8 * j + 0], f[8 * j + 1]);
            __nv_bfloat162 p1 = __floats2bfloat162_rn(f[8 * j + 2], f[8 * j + 3]);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(f[8 * j + 4], f[8 * j + 5]);
            __nv_bfloat162 p3 = __floats2bfloat162_rn(f[8 * j + 6], f[8 * j + 7]);
            uint4 u;
            u.x = *reinterpret_cast<uint32_t *>(&p0);
            u.y = *reinterpret_cast<uint32_t *>(&p1);
            u.z = *reinterpret_cast<uint32_t *>(&p2);
            u.w = *reinterpret_cast<uint32_t *>(&p3);
            *reinterpret_cast<uint4 *>(srow + off + 16 * j) = u;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4 *>(srow + off + 16 * j) =
                make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
    }
}

template <bool kOutBF16>
__global__ void __launch_bounds__(kGemmThreads, 1)
    patch_embed_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const float *__restrict__ bias, void *__restrict__ out, int64_t M, int32_t N, int32_t K,
                       int32_t *__restrict__ err, uint32_t wait_limit, int32_t stop_after) {
    extern __shared__ __align__(1024) uint8_t gemm_smem_raw[];
    // 1024-byte aligned tiles (the swizzle pattern repeats every 1024 bytes); the
    // offset is the same in both CTAs, as the pair MMA requires
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ GemmSmem S;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();     // 0: even CTA (issues the MMAs), 1: its peer
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
    const int n_tiles = N / kBN;
    const int64_t m_tiles = (M + kPairM - 1) / kPairM;
    const int64_t total_tiles = m_tiles * n_tiles;
    const int kblocks = K / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_free[b], 2 * kEpiWarps);
        }
        mbar_init(&S.drain, 1);
        S.failed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = S.tmem_base;

    if (warp == 0 || warp == 6) {
        // ---- producers (both CTAs): warp 0 this CTA's half of A, warp 6 its half of B; the
        // k-block counter g runs across tiles
        const bool loads_a = warp == 0;
        if (lane == 0) {
            uint32_t g = 0;
            for (int64_t t = pair; t < total_tiles && !stopped(S); t += pairs) {
                const int a_row = static_cast<int>((t / n_tiles) * kPairM) + static_cast<int>(rank) * kBM;
                const int b_row = static_cast<int>(t % n_tiles) * kBN + static_cast<int>(rank) * kBNHalf;
                for (int kb = 0; kb < kblocks; ++kb, ++g) {
                    // test hook: a loader that stops after `stop_after` k blocks (never in normal launches)
                    if (stop_after >= 0 && g >= static_cast<uint32_t>(stop_after)) break;
                    const uint32_t s = g % kStages, use = g / kStages;
                    if (use > 0 && !mbar_wait(&S.empty[s], (use - 1) & 1, wait_limit)) {
                        fail(S, err, kErrEmptyWait);
                        break;
                    }
                    if (stopped(S)) break;
                    uint8_t *a = tiles + s * kStageBytes;
                    const uint32_t full_bar = cluster_addr(&S.full[s], 0);
                    // The B bytes may land before the expectation is posted: the transaction count of
                    // the phase goes negative for a while, and the phase cannot complete before the
                    // single arrival below.
                    if (loads_a) {
                        if (leader) mbar_expect_tx(&S.full[s], 2 * kStageBytes);  // both CTAs, A and B
                        tma_load_2d_pair(a, &map_a, full_bar, kb * kBK, a_row);
                        tma_load_2d_pair(a + kAAtomBytes, &map_a, full_bar, kb * kBK + kAtomK, a_row);
                    } else {
                        uint8_t *b = a + kATileBytes;
                        tma_load_2d_pair(b, &map_b, full_bar, kb * kBK, b_row);
                        tma_load_2d_pair(b + kBAtomBytes, &map_b, full_bar, kb * kBK + kAtomK, b_row);
                    }
                }
            }
            // copies still in flight land before the CTA can leave (bounded; the even
            // CTA's barrier counts the B loader's and the peer's copies as well)
            if (leader && loads_a)
                for (uint32_t q = (g > kStages ? g - kStages : 0); q < g; ++q)
                    mbar_wait(&S.full[q % kStages], (q / kStages) & 1, wait_limit);
        }
    } else if (warp == 1) {
        // ---- MMA issuer: one lane of the even CTA drives the tensor cores of both SMs
        if (leader && lane == 0) {
            uint32_t g = 0, i = 0;
            for (int64_t t = pair; t < total_tiles && !stopped(S); t += pairs, ++i) {
                const uint32_t b = i & 1, use_b = i >> 1;
                if (use_b > 0 && !mbar_wait(&S.acc_free[b], (use_b - 1) & 1, wait_limit)) {
                    fail(S, err, kErrAccumFreeWait);
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t acc = tmem + b * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb, ++g) {
                    const uint32_t s = g % kStages;
                    if (!mbar_wait(&S.full[s], (g / kStages) & 1, wait_limit)) {
                        fail(S, err, kErrFullWait);
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t a = smem_u32(tiles + s * kStageBytes);
                    const uint32_t bb = a + kATileBytes;
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k) {
                        // 64-wide half k / 4, then 16 bf16 (32 bytes) at a time inside its swizzled 128-byte rows
                        const int h = k / (kAtomK / kUmmaK), kk = k % (kAtomK / kUmmaK);
                        const uint64_t da = kmajor_sw128_desc(a + h * kAAtomBytes + kk * kUmmaK * 2);
                        const uint64_t db = kmajor_sw128_desc(bb + h * kBAtomBytes + kk * kUmmaK * 2);
                        const uint32_t accumulate = (kb > 0 || k > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred p;\n\t"
                            "setp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(acc),
                            "l"(da), "l"(db), "r"(kInstrDesc), "r"(accumulate)
                            : "memory");
                    }
                    umma_commit_pair(&S.empty[s]);  // stage s is free in both CTAs once these MMAs have read it
                }
                if (!ok) break;
                umma_commit_pair(&S.acc_full[b]);
            }
            // every MMA issued has finished before TMEM can be freed (bounded)
            umma_commit_local(&S.drain);
            if (!mbar_wait(&S.drain, 0, wait_limit)) fail(S, err, kErrDrainWait);
        }
    } else if (warp <= 5) {
        // ---- epilogue (both CTAs): warp w reads TMEM lanes 32*(w % 4) .. +31 (its accessible quarter)
        const int quarter = warp & 3;
        uint8_t *stage = tiles + kStages * kStageBytes + (warp - 2) * kEpiStageBytes;
        uint32_t i = 0;
        for (int64_t t = pair; t < total_tiles; t += pairs, ++i) {
            const uint32_t b = i & 1;
            // uniform across the warp: tcgen05.ld below is a warp-wide instruction
            const bool ready =
                __all_sync(0xffffffffu, !stopped(S) && mbar_wait(&S.acc_full[b], (i >> 1) & 1, wait_limit));
            if (!ready) {
                if (lane == 0) fail(S, err, kErrAccumWait);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // rows of this warp: row0 .. row0 + 31; lane `lane` holds row row0 + lane in TMEM
            const int64_t row0 = (t / n_tiles) * kPairM + rank * kBM + quarter * 32;
            const int n0 = static_cast<int>(t % n_tiles) * kBN;
            const uint32_t base = tmem + b * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
            // one output line (128 bytes) per row at a time: 64 bf16 or 32 fp32 columns
            constexpr int kLineCols = kOutBF16 ? 64 : 32;
            constexpr int kEsz = kOutBF16 ? 2 : 4;
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += kLineCols) {
                uint32_t v[32];
                tmem_ld32(base + static_cast<uint32_t>(c0), v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                stage_32<kOutBF16>(stage + lane * kStagePitch, 0, v, bias, n0 + c0);
                if constexpr (kOutBF16) {
                    tmem_ld32(base + static_cast<uint32_t>(c0 + 32), v);
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    stage_32<kOutBF16>(stage + lane * kStagePitch, 64, v, bias, n0 + c0 + 32);
                }
                if (c0 + kLineCols == kBN) {
                    // the whole accumulator has been read: hand it back to the MMA lane
                    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(cluster_addr(&S.acc_free[b], 0));
                }
                __syncwarp();
                // 8 lanes per row: each store instruction writes 4 whole 128-byte lines
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = i * 4 + (lane >> 3);
                    const int64_t row = row0 + r;
                    const uint4 u = *reinterpret_cast<const uint4 *>(stage + r * kStagePitch + (lane & 7) * 16);
                    if (row < M)
                        __stcs(reinterpret_cast<uint4 *>(static_cast<uint8_t *>(out) +
                                                         (row * N + n0 + c0) * kEsz + (lane & 7) * 16),
                               u);
                }
                __syncwarp();
            }
        }
    }

    // both CTAs stay until the pair is done with each other's barriers, shared
    // memory and TMEM; then each frees its TMEM
    __syncwarp();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 row-major [rows, cols] map with a box of box_rows x 64 columns,
// 128-byte swizzle; rows past the end read as zero.
bool make_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kAtomK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_patch_embed(const void *d_rows, int64_t M, int32_t K, const void *d_weight, int32_t N, const float *d_bias,
                       int32_t out_dtype, void *d_out, int32_t *d_err, void *stream, uint32_t wait_rounds,
                       int32_t stop_after) {
    const uint32_t wait_limit = wait_rounds ? wait_rounds : kWaitLimit;
    CUtensorMap ma, mb;
    if (!make_map(&ma, d_rows, M, K, kBM) || !make_map(&mb, d_weight, N, K, kBNHalf)) return MIMO_ECUDA;
    const int64_t tiles = ((M + kPairM - 1) / kPairM) * (N / kBN);
    const size_t smem = static_cast<size_t>(kStages) * kStageBytes + kEpiWarps * kEpiStageBytes + 1024;
    const int out_bf16 = out_dtype == MIMO_BF16 ? 1 : 0;
    auto kernel = out_bf16 ? patch_embed_kernel<true> : patch_embed_kernel<false>;
    // per host thread and device: the shared-memory opt-in and the number of
    // resident CTA pairs, looked up on the first launch (a chained call
    // launches this kernel once per run of images)
    struct Setup {
        int max_pairs[2] = {0, 0};
    };
    constexpr int kMaxDevices = 64;
    static thread_local Setup setup_of[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MIMO_ECUDA;
    int &max_pairs = setup_of[dev].max_pairs[out_bf16];
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as can be resident at once (one CTA per SM)
    if (max_pairs < 1) {
        int sms = 0, found = 0;
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
            return MIMO_ECUDA;
        cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
        if (cudaOccupancyMaxActiveClusters(&found, kernel, &cfg) != cudaSuccess || found < 1) return MIMO_ECUDA;
        max_pairs = found;
    }
    const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    if (cudaLaunchKernelEx(&cfg, kernel, ma, mb, d_bias, d_out, M, N, K, d_err, wait_limit, stop_after) !=
        cudaSuccess)
        return MIMO_ECUDA;
    return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ECUDA;
}

}  // namespace mimo
