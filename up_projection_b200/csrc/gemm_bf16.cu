// gemm_bf16.cu -- fused SwiGLU dual GEMM for bf16, sm_100a.
//
//   H[m, n] = silu(sum_k X[m,k] Wg[n,k]) * (sum_k X[m,k] Wu[n,k])
//
// The "dual gemm with activations" of Liger-Kernel issue #937 (approach 3),
// written for Blackwell's 5th-generation tensor cores:
//
//  * one CTA per SM, persistent over 128 x 128 output tiles;
//  * warp 0 (one thread): TMA producer.  Per 64-deep k-block it loads the X
//    tile [128 x 64] once and the Wg and Wu tiles [128 x 64] stacked into one
//    256-row B tile, into a 4-stage shared-memory ring (128-byte swizzle);
//  * warp 1 (one thread): MMA issuer.  One tcgen05.mma (M=128, N=256, K=16)
//    per 16-deep step multiplies the shared X tile by the stacked [Wg; Wu]
//    tile, so both projections share one read of X from shared memory and
//    the accumulator holds the gate in columns 0..127 and the up projection
//    in columns 128..255 (fp32, in tensor memory).  The accumulator is double
//    buffered (2 x 256 of the 512 TMEM columns) so the next tile's MMAs run
//    while the epilogue drains the previous one;
//  * warps 2..5: epilogue.  tcgen05.ld brings matching gate/up columns of a
//    row into registers, h = g * sigmoid(g) * u is formed in fp32 on the
//    accumulators (no intermediate rounding, as the numerics note of
//    TensorRT-LLM PR #17693 describes for a fused epilogue), rounded once to
//    bf16, written to a swizzled staging buffer and stored by TMA.  G and U
//    never reach global memory.
//
// Pair mode (M > 128): each MMA covers 256 rows over the two CTAs of a
// cluster (tcgen05 cta_group::2); a CTA holds its own 128 rows of X and half
// of the stacked weight rows -- the even CTA the tile's Wg rows, the odd one
// its Wu rows -- so each SM loads and reads 32 KB per stage instead of 48;
// both CTAs' copies are counted on the even CTA's barrier, whose warp 1
// issues the pair's MMAs and commits to the barriers of both CTAs, and each
// CTA's epilogue drains its own 128 accumulator rows.  (B200, LLaMA-3 8B
// shapes: the same speed at M = 8192 and 4096, +2.4 % at M = 1024, +10 % at
// M = 256: the single-SM kernel is not bound by shared-memory traffic, as
// the fp32 one is.)
//
// Edge tiles: TMA zero-fills rows/columns/k beyond the tensor on load and
// clips the store.  Every wait is bounded (ptx.cuh): a stuck pipeline sets
// the status word and the kernel returns after releasing what it holds.
#include <cuda_bf16.h>

#include <atomic>

#include "activation.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace swiglu {

// Status word of this translation unit's kernel; bit 0 = a bounded wait
// gave up.  Read and cleared by gemm_bf16_status_fetch_and_clear().
__device__ unsigned int g_gemm_bf16_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;
using gemm::tile_coords;

constexpr int kBM = 128;                // rows of X per CTA and tile (= MMA M per SM)
constexpr int kBN = 128;                // columns of H per tile (gate, up each)
constexpr int kBK = 64;                 // k per stage: one 128-byte bf16 row
constexpr int kUmmaK = 16;              // k per tcgen05.mma, kind::f16
constexpr int kAccCols = 2 * kBN;       // TMEM columns per accumulator buffer
constexpr int kTmemCols = 2 * kAccCols; // double buffered: all 512 columns
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kABytes = kBM * kBK * 2;           // 16 KB
constexpr uint32_t kEpiBufBytes = 32 * 128;           // 32 rows x 64 bf16

// Shared-memory layout of one CTA.  kPair: each MMA covers 256 rows over the
// two CTAs of a cluster (tcgen05 cta_group::2); a CTA then holds its own 128
// rows of X and half of the stacked weight rows -- the even CTA the tile's
// 128 Wg rows, the odd one its 128 Wu rows -- so a stage is 32 KB, not 48.
template <bool kPair>
struct Layout {
    static constexpr int kStages = kPair ? 6 : 4;
    static constexpr uint32_t kBBytes = (kPair ? 1 : 2) * kBN * kBK * 2;  // Wg [and Wu] rows
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + kStages * kABytes;
    static constexpr uint32_t kOffEpi = kOffB + kStages * kBBytes;
    static constexpr uint32_t kOffBar = kOffEpi + kEpiWarps * kEpiBufBytes;
    static constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1;  // full, empty, tfull, tempty, drain
    static constexpr uint32_t kOffTmemPtr = kOffBar + 8 * kNumBars;
    static constexpr uint32_t kOffAbort = kOffTmemPtr + 8;
    static constexpr uint32_t kSmemUsed = kOffAbort + 8;
    static constexpr uint32_t kSmemBytes = kSmemUsed + 1024;       // slack for 1024-B alignment
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB opt-in shared memory");
};

static_assert(kBN % 64 == 0, "epilogue works in 64-column chunks");

__device__ __forceinline__ float gated_fast(int which, float alpha, uint32_t gbits,
                                            uint32_t ubits) {
    return act::gated<false>(which, alpha, __uint_as_float(gbits), __uint_as_float(ubits));
}

// fp8 output of one (1,32) block held by this lane: h = act(alpha g) u for
// the 32 accumulator pairs, amax, the UE8M0 exponent e = the smallest
// integer with amax <= 448 * 2^e (clamped to [-127, 127]), and the e4m3
// codes of h / 2^e (round to nearest even; |h / 2^e| <= 448, so the
// saturating conversion never saturates a finite block).  A block holding
// Inf or NaN gets scale code 0xFF and NaN codes.  Returns the scale code;
// q receives the 32 codes, 4 per word, column order.
__device__ __forceinline__ uint32_t quant_block_e4m3(int which, float alpha, const uint32_t (&g)[32],
                                                    const uint32_t (&u)[32], uint32_t (&q)[8]) {
    float h[32];
    float amax = 0.0f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        h[i] = gated_fast(which, alpha, g[i], u[i]);
        finite = finite && ((__float_as_uint(h[i]) & 0x7f800000u) != 0x7f800000u);
        amax = fmaxf(amax, fabsf(h[i]));
    }
    if (!finite) {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = 0x7f7f7f7fu;
        return 0xFFu;
    }
    const uint32_t bits = __float_as_uint(amax);
    const int ef = static_cast<int>(bits >> 23);          // amax >= 0
    int e = -127;
    if (ef != 0) {
        // amax = 1.f * 2^(ef-127) <= 1.75 * 2^(e+8)
        e = (ef - 127) - 8 + ((bits & 0x7fffffu) > 0x600000u ? 1 : 0);
        e = max(-127, min(127, e));
    }
    // h * 2^-e as two exact power-of-two products (each factor normal)
    const int n1 = (-e) / 2, n2 = -e - n1;
    const float s1 = __uint_as_float(static_cast<uint32_t>(127 + n1) << 23);
    const float s2 = __uint_as_float(static_cast<uint32_t>(127 + n2) << 23);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        // cvt ... d, a, b puts a in the upper byte: column order in memory
        unsigned short lo, hi;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(lo)
            : "f"(h[4 * i + 1] * s1 * s2), "f"(h[4 * i] * s1 * s2));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(hi)
            : "f"(h[4 * i + 3] * s1 * s2), "f"(h[4 * i + 2] * s1 * s2));
        q[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    return static_cast<uint32_t>(e + 127);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
    swiglu_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_x,
                            const __grid_constant__ CUtensorMap tm_wg,
                            const __grid_constant__ CUtensorMap tm_wu,
                            const __grid_constant__ CUtensorMap tm_h,
                            const __grid_constant__ CUtensorMap tm_g,
                            const __grid_constant__ CUtensorMap tm_u, int M, int N, int K,
                            int num_m_tiles, int num_n_tiles, int which_act, float alpha,
                            int store_gu, uint8_t *__restrict__ scales) {
    using L = Layout<kPair>;
    constexpr int kStages = L::kStages;
    constexpr uint32_t kBBytes = L::kBBytes;
    constexpr uint32_t kStageBytes = L::kStageBytes;
    constexpr uint32_t kOffA = L::kOffA, kOffB = L::kOffB, kOffEpi = L::kOffEpi;
    constexpr uint32_t kOffBar = L::kOffBar, kOffTmemPtr = L::kOffTmemPtr, kOffAbort = L::kOffAbort;
    constexpr int kGroup = kPair ? gemm::kGroupMForward / 2 : gemm::kGroupMForward;
    constexpr int kRowsPerTile = kPair ? 2 * kBM : kBM;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const uint32_t sa = base + kOffA;
    const uint32_t sb = base + kOffB;
    const uint32_t se = base + kOffEpi;
    const uint32_t bar_full = base + kOffBar;
    const uint32_t bar_empty = bar_full + 8 * kStages;
    const uint32_t bar_tfull = bar_empty + 8 * kStages;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t bar_drain = bar_tempty + 16;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(gbase + kOffTmemPtr);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + kOffAbort);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int num_tiles = num_m_tiles * num_n_tiles;   // kPair: 256-row tiles
    const int num_kb = (K + kBK - 1) / kBK;
    // kPair: CTA `rank` of pair `unit`; rank 0 issues the pair's MMAs
    const uint32_t rank = kPair ? cluster_rank() : 0u;
    const int unit = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
    const int units = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, (kPair ? 2 : 1) * kEpiWarps);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        if (!kPair || rank == 0) tma_prefetch_desc(&tm_wg);
        if (!kPair || rank == 1) tma_prefetch_desc(&tm_wu);
        tma_prefetch_desc(&tm_h);
        if (store_gu) {
            tma_prefetch_desc(&tm_g);
            tma_prefetch_desc(&tm_u);
        }
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(smem_u32(tmem_ptr), kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_ptr), kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (kPair) {
        // both CTAs' barriers initialised and TMEM allocated before any
        // copy, arrive or MMA that reaches the other CTA
        cluster_sync_all();
    } else {
        __syncthreads();
    }
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_ptr);

    bool failed = false;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            // kPair: every copy of both CTAs is counted on the even CTA's
            // full barrier, whose producer expects the pair's bytes
            const uint32_t full_r0 = kPair ? map_to_rank(bar_full, 0) : 0u;
            const CUtensorMap *tm_w = rank == 0 ? &tm_wg : &tm_wu;
            for (int t = unit; t < num_tiles && !failed; t += units) {
                int mt, nt;
                tile_coords<kGroup>(t, num_m_tiles, num_n_tiles, mt, nt);
                const int m0 = mt * kRowsPerTile + static_cast<int>(rank) * kBM, n0 = nt * kBN;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t a_dst = sa + stage * kABytes;
                    const uint32_t b_dst = sb + stage * kBBytes;
                    if constexpr (kPair) {
                        if (rank == 0) mbar_arrive_expect_tx(fb, 2 * kStageBytes);
                        const uint32_t fb_r0 = full_r0 + 8 * stage;
                        tma_load_2d_pair(&tm_x, fb_r0, a_dst, kb * kBK, m0);
                        tma_load_2d_pair(tm_w, fb_r0, b_dst, kb * kBK, n0);
                    } else {
                        mbar_arrive_expect_tx(fb, kStageBytes);
                        tma_load_2d(&tm_x, fb, a_dst, kb * kBK, m0);
                        tma_load_2d(&tm_wg, fb, b_dst, kb * kBK, n0);
                        tma_load_2d(&tm_wu, fb, b_dst + kBBytes / 2, kb * kBK, n0);
                    }
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Never leave while a load issued here may still write shared
            // memory.  (kPair: the even CTA's full barriers count the copies
            // of both CTAs; the odd CTA's copies are consumed by the pair's
            // MMAs before the final cluster barrier.)
            for (int s = 0; s < kStages && (!kPair || rank == 0); ++s) {
                if (issued > s) {
                    const long long uses = (issued - 1 - s) / kStages + 1;
                    mbar_wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = make_idesc(1u, kRowsPerTile, 2 * kBN);
            // kPair: the odd CTA's barriers, as addresses in the cluster window
            const uint32_t empty_r1 = kPair ? map_to_rank(bar_empty, 1) : 0u;
            const uint32_t tfull_r1 = kPair ? map_to_rank(bar_tfull, 1) : 0u;
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = unit; t < num_tiles && !failed; t += units) {
                if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = sw128_kmajor_desc(sa + stage * kABytes);
                    const uint64_t bdesc = sw128_kmajor_desc(sb + stage * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                        // +32 bytes along K inside the swizzled row = +2 in the
                        // descriptor's start-address field.
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        if constexpr (kPair)
                            mma_f16_pair(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, accum);
                        else
                            mma_f16(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, accum);
                    }
                    if constexpr (kPair) {
                        // the stage is free in both CTAs
                        mma_commit_pair(bar_empty + 8 * stage);
                        mma_commit_pair(empty_r1 + 8 * stage);
                    } else {
                        mma_commit(bar_empty + 8 * stage);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (failed) break;
                if constexpr (kPair) {
                    mma_commit_pair(bar_tfull + 8 * acc);
                    mma_commit_pair(tfull_r1 + 8 * acc);
                } else {
                    mma_commit(bar_tfull + 8 * acc);
                }
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Every MMA issued here must finish before TMEM is released.
            if constexpr (kPair)
                mma_commit_pair(bar_drain);
            else
                mma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0);
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may read
        const uint32_t row_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t buf = se + static_cast<uint32_t>(warp - 2) * kEpiBufBytes;
        const uint32_t swz = static_cast<uint32_t>(lane & 7);
        // kPair: the accumulator is released on the even CTA's barrier
        const uint32_t tempty_r0 = kPair ? map_to_rank(bar_tempty, 0) : 0u;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = unit; t < num_tiles; t += units) {
            int mt, nt;
            tile_coords<kGroup>(t, num_m_tiles, num_n_tiles, mt, nt);
            const int m0 = mt * kRowsPerTile + static_cast<int>(rank) * kBM, n0 = nt * kBN;
            if (!mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem_base + row_off + static_cast<uint32_t>(acc * kAccCols);
            if (scales != nullptr) {
                // fp8 output: the lane's row, one (1,32) block per 32 columns.
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
                const int row = m0 + quad * 32 + lane;
                const int nblk = (N + 31) / 32;
#pragma unroll 1
                for (int b = 0; b < kBN / 32; ++b) {
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(tacc + 32u * b, g);
                    tmem_ld_32x32b_x32(tacc + kBN + 32u * b, u);
                    tmem_ld_wait(g);
                    tmem_ld_wait(u);
                    uint32_t q[8];
                    const uint32_t code = quant_block_e4m3(which_act, alpha, g, u, q);
                    sts_v4(buf + static_cast<uint32_t>(lane) * 128u +
                               ((static_cast<uint32_t>(2 * b) ^ swz) << 4),
                           make_uint4(q[0], q[1], q[2], q[3]));
                    sts_v4(buf + static_cast<uint32_t>(lane) * 128u +
                               ((static_cast<uint32_t>(2 * b + 1) ^ swz) << 4),
                           make_uint4(q[4], q[5], q[6], q[7]));
                    const int cb = n0 / 32 + b;
                    if (row < M && cb < nblk)
                        scales[static_cast<long long>(row) * nblk + cb] = static_cast<uint8_t>(code);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int y = m0 + quad * 32;
                    if (n0 < N && y < M) {
                        tma_store_2d(&tm_h, buf, n0, y);
                        bulk_commit();
                    }
                }
            }
            // Per 64-column chunk: H = act(alpha g) u, then (training
            // forward) G and U themselves, each staged and stored by TMA.
            const int outputs = scales != nullptr ? 0 : (store_gu ? 3 : 1);
#pragma unroll 1
            for (int c = 0; c < (outputs ? kBN / 64 : 0); ++c) {
#pragma unroll 1
                for (int what = 0; what < outputs; ++what) {
                    // The previous store from this buffer must have read it.
                    if (lane == 0) bulk_wait_read<0>();
                    __syncwarp();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t g[32], u[32];
                        const uint32_t col = static_cast<uint32_t>(c * 64 + h * 32);
                        if (what != 2) tmem_ld_32x32b_x32(tacc + col, g);
                        if (what != 1) tmem_ld_32x32b_x32(tacc + kBN + col, u);
                        tmem_ld_wait(g);
                        tmem_ld_wait(u);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 v;
                            uint32_t *pv = &v.x;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int e = 8 * j + 2 * q;
                                if (what == 0)
                                    pv[q] = pack_bf16x2(gated_fast(which_act, alpha, g[e], u[e]),
                                                        gated_fast(which_act, alpha, g[e + 1], u[e + 1]));
                                else if (what == 1)
                                    pv[q] = pack_bf16x2(__uint_as_float(g[e]), __uint_as_float(g[e + 1]));
                                else
                                    pv[q] = pack_bf16x2(__uint_as_float(u[e]), __uint_as_float(u[e + 1]));
                            }
                            // 16-byte chunk (h*4 + j) of this lane's 128-byte row,
                            // placed where the TMA 128-byte swizzle expects it.
                            const uint32_t chunk = static_cast<uint32_t>(h * 4 + j);
                            sts_v4(buf + static_cast<uint32_t>(lane) * 128u + ((chunk ^ swz) << 4), v);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int x = n0 + c * 64;
                        const int y = m0 + quad * 32;
                        if (x < N && y < M) {
                            const CUtensorMap *dst = what == 0 ? &tm_h : (what == 1 ? &tm_g : &tm_u);
                            tma_store_2d(dst, buf, x, y);
                            bulk_commit();
                        }
                    }
                }
            }
            // All tcgen05.ld of this buffer have completed (waited above).
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (kPair)
                    mbar_arrive_remote(tempty_r0 + 8 * acc);
                else
                    mbar_arrive(bar_tempty + 8 * acc);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait<0>();
    }

    if (failed) atomicOr(&g_gemm_bf16_status, 1u);

    tc_fence_before();
    __syncthreads();
    // kPair: the pair's MMAs have completed (the issuer drained them) and
    // both epilogues are done before either CTA frees TMEM or leaves
    if constexpr (kPair) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        __syncwarp();
        if constexpr (kPair)
            tmem_dealloc_pair(tmem_base, kTmemCols);
        else
            tmem_dealloc(tmem_base, kTmemCols);
    }
}

std::atomic<unsigned> g_attr_set_mask[2];

}  // namespace

cudaError_t launch_gemm_bf16(const void *X, const void *Wg, const void *Wu, void *H, int M,
                             int K, int N, const Epilogue &epi, const DeviceInfo &dev,
                             cudaStream_t stream) {
    CUtensorMap tx, twg, twu, th, tg, tu;
    const CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const bool store_gu = epi.G != nullptr;
    const bool fp8 = epi.scales != nullptr;
    // fp8 output: H is [M, N] bytes stored in 128-column boxes.
    const bool h_ok = fp8 ? encode_tmap_2d(&th, H, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, M,
                                           static_cast<uint64_t>(N), 128, 32, sw)
                          : encode_tmap_2d(&th, H, bf16, N, M, static_cast<uint64_t>(N) * 2, 64,
                                           32, sw);
    if (!h_ok || !encode_tmap_2d(&tx, X, bf16, K, M, static_cast<uint64_t>(K) * 2, kBK, kBM, sw) ||
        !encode_tmap_2d(&twg, Wg, bf16, K, N, static_cast<uint64_t>(K) * 2, kBK, kBN, sw) ||
        !encode_tmap_2d(&twu, Wu, bf16, K, N, static_cast<uint64_t>(K) * 2, kBK, kBN, sw) ||
        !encode_tmap_2d(&tg, store_gu ? epi.G : H, bf16, N, M, static_cast<uint64_t>(N) * 2, 64, 32,
                        sw) ||
        !encode_tmap_2d(&tu, store_gu ? epi.U : H, bf16, N, M, static_cast<uint64_t>(N) * 2, 64, 32,
                        sw)) {
        return cudaErrorInvalidValue;
    }
    const int num_n = (N + kBN - 1) / kBN;
    const int store = store_gu ? 1 : 0;
    uint8_t *sc = static_cast<uint8_t *>(epi.scales);
    const unsigned bit = 1u << (dev.device & 31);
    if (M > kBM) {
        // pairs of SMs: tiles of 256 rows, a cluster of two CTAs per tile
        auto kernel = swiglu_gemm_bf16_kernel<true>;
        if (!(g_attr_set_mask[1].load() & bit)) {
            cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(Layout<true>::kSmemBytes));
            if (e != cudaSuccess) return e;
            g_attr_set_mask[1].fetch_or(bit);
        }
        const int num_m2 = (M + 2 * kBM - 1) / (2 * kBM);
        const long long tiles = static_cast<long long>(num_m2) * num_n;
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = Layout<true>::kSmemBytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(2);
        int max_clusters = 0;
        cudaError_t e = cudaOccupancyMaxActiveClusters(&max_clusters, kernel, &cfg);
        if (e != cudaSuccess) return e;
        if (max_clusters < 1) return cudaErrorInvalidConfiguration;
        const long long pairs = tiles < max_clusters ? tiles : max_clusters;
        cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
        e = cudaLaunchKernelEx(&cfg, kernel, tx, twg, twu, th, tg, tu, M, N, K, num_m2, num_n,
                               epi.activation, epi.gate_multiplier, store, sc);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    if (!(g_attr_set_mask[0].load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(swiglu_gemm_bf16_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(Layout<false>::kSmemBytes));
        if (e != cudaSuccess) return e;
        g_attr_set_mask[0].fetch_or(bit);
    }
    const int num_m = (M + kBM - 1) / kBM;
    const long long tiles = static_cast<long long>(num_m) * num_n;
    const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
    swiglu_gemm_bf16_kernel<false><<<grid, kThreads, Layout<false>::kSmemBytes, stream>>>(
        tx, twg, twu, th, tg, tu, M, N, K, num_m, num_n, epi.activation, epi.gate_multiplier,
        store, sc);
    return cudaGetLastError();
}

cudaError_t gemm_bf16_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_gemm_bf16_status, sizeof(unsigned int),
                                              0, cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gemm_bf16_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
