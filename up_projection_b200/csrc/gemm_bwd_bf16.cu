// gemm_bwd_bf16.cu -- the two GEMMs of the projection's backward pass, bf16,
// sm_100a.  With G = X Wg^T, U = X Wu^T and dG, dU from dSwiGLU:
//
//   dX  [M,K] = dG Wg + dU Wu                  (reduction over N)
//   dWg [N,K] = dG^T X,   dWu [N,K] = dU^T X    (reduction over M)
//
// the backward half of the fused MLP's forward/backward dataflow (page
// "[RFC] Testing Methodology for FP32 Convergence Tests on Fused
// SwiGLU/dSwiGLU Kernels", Background).
//
// One kernel template serves both, with the forward's persistent
// warp-specialised skeleton (TMA producer warp, single-thread tcgen05.mma
// issuer, four epilogue warps, double-buffered fp32 accumulators in TMEM):
//
//  * dX: one output tile [128 x BN] accumulates BOTH products in one TMEM
//    accumulator -- the reduction runs over the 2N columns of [dG | dU]
//    against the 2N rows of [Wg ; Wu], switching tensor maps half way, so
//    dX is formed and rounded once.  A (dG, dU) is K-major like the forward's
//    X; B (Wg, Wu, whose contiguous index is the output column) is MN-major.
//  * dW: the output is [dWg ; dWu] seen as one [2N x K] matrix; a row tile
//    belongs to dWg or dWu and reads the matching gradient.  Both operands are
//    MN-major: A = dG^T / dU^T (n contiguous in dG), B = X (k contiguous).
//    Row tiles of dWg and dWu over the same columns share X through L2
//    (they are rastered together); one MMA of N = BN per 16-deep step keeps
//    the shared-memory operand traffic at the forward's 12 KB per MFLOP.
//
// MN-major tiles are TMA boxes {64, 64} in the 128-byte swizzle, one per
// 64-wide MN atom; the UMMA descriptor walks atoms with its leading byte
// offset (ptx.cuh).  Out-of-range rows/columns/reduction steps are
// zero-filled by TMA on load and clipped on store, so any M, N, K that are
// multiples of 8 (16-byte rows) work, with ragged tails.  Every wait is
// bounded: a stuck pipeline sets the status word and the kernel returns
// after releasing what it holds.
#include <cuda_bf16.h>

#include <atomic>

#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace swiglu {

// Bit 0: a bounded wait gave up.  Read by gemm_bwd_status_fetch_and_clear().
__device__ unsigned int g_gemm_bwd_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;
using gemm::tile_coords;

enum : int { kModeDx = 0, kModeDw = 1 };

constexpr int kBM = 128;             // output rows per tile (= MMA M)
constexpr int kBR = 64;              // reduction depth per stage (128-byte rows)
constexpr int kUmmaK = 16;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kAtomBytes = 64 * kBR * 2;   // MN-major atom: 64 x 64 bf16 = 8 KB
constexpr uint32_t kABytes = kBM * kBR * 2;     // 16 KB either way
constexpr uint32_t kEpiBufBytes = 32 * 128;     // 32 rows x 64 bf16
constexpr uint32_t kRingBudget = 200 * 1024;

template <int kBN>
struct Cfg {
    static constexpr uint32_t kBBytes = kBN * kBR * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = static_cast<int>(kRingBudget / kStageBytes);
    // Double-buffered accumulator; allocations are powers of two.
    static constexpr int kTmemCols = 2 * kBN <= 256 ? 256 : 512;
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + kStages * kABytes;
    static constexpr uint32_t kOffEpi = kOffB + kStages * kBBytes;
    static constexpr uint32_t kOffBar = kOffEpi + kEpiWarps * kEpiBufBytes;
    static constexpr uint32_t kNumBars = 2 * kStages + 2 + 2 + 1;
    static constexpr uint32_t kOffTmemPtr = kOffBar + 8 * kNumBars;
    static constexpr uint32_t kOffAbort = kOffTmemPtr + 8;
    static constexpr uint32_t kSmemBytes = kOffAbort + 8 + 1024;
    static_assert(kBN == 128 || kBN == 192 || kBN == 256, "whole 64-wide atoms, MMA N <= 256");
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB opt-in shared memory");
};

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<uint32_t *>(&v);
}

// Problem geometry shared by the three roles.
//   dX: rows = M, red = N per pair (two pairs), row tiles ceil(M/128)
//   dW: rows = N per matrix (two matrices), red = M, row tiles 2 ceil(N/128)
struct Geo {
    int rows;        // output rows of one output matrix
    int cols;        // output columns (K)
    int row_tiles;   // row tiles of one output matrix
    int num_m;       // row tiles in the raster
    int num_n;       // column tiles
    int kb_pair;     // 64-deep reduction blocks of one pair
};

template <int kMode, int kBN>
__global__ void __launch_bounds__(kThreads, 1)
    swiglu_gemm_bwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_a0,
                                const __grid_constant__ CUtensorMap tm_a1,
                                const __grid_constant__ CUtensorMap tm_b0,
                                const __grid_constant__ CUtensorMap tm_b1,
                                const __grid_constant__ CUtensorMap tm_o0,
                                const __grid_constant__ CUtensorMap tm_o1, Geo geo) {
    using C = Cfg<kBN>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const uint32_t sa = base + C::kOffA;
    const uint32_t sb = base + C::kOffB;
    const uint32_t se = base + C::kOffEpi;
    const uint32_t bar_full = base + C::kOffBar;
    const uint32_t bar_empty = bar_full + 8 * C::kStages;
    const uint32_t bar_tfull = bar_empty + 8 * C::kStages;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t bar_drain = bar_tempty + 16;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(gbase + C::kOffTmemPtr);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + C::kOffAbort);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int num_tiles = geo.num_m * geo.num_n;
    const int num_kb = kMode == kModeDx ? 2 * geo.kb_pair : geo.kb_pair;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, kEpiWarps);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_a0);
        tma_prefetch_desc(&tm_a1);
        tma_prefetch_desc(&tm_b0);
        tma_prefetch_desc(&tm_b1);
        tma_prefetch_desc(&tm_o0);
        tma_prefetch_desc(&tm_o1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_ptr);

    bool failed = false;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int t = blockIdx.x; t < num_tiles && !failed; t += gridDim.x) {
                int mt, nt;
                tile_coords(t, geo.num_m, geo.num_n, mt, nt);
                const int c0 = nt * kBN;
                // dW: which matrix this row tile belongs to, and its first row.
                const int second = (kMode == kModeDw && mt >= geo.row_tiles) ? 1 : 0;
                const int r0 = (mt - second * geo.row_tiles) * kBM;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t a_dst = sa + stage * kABytes;
                    const uint32_t b_dst = sb + stage * C::kBBytes;
                    mbar_arrive_expect_tx(fb, C::kStageBytes);
                    if (kMode == kModeDx) {
                        const int pair = kb >= geo.kb_pair ? 1 : 0;
                        const int red0 = (kb - pair * geo.kb_pair) * kBR;
                        // A: [128 rows of dG or dU] x [64 of N], K-major.
                        tma_load_2d(pair ? &tm_a1 : &tm_a0, fb, a_dst, red0, r0);
                        // B: [64 rows of Wg or Wu] x [BN of K], MN-major atoms.
#pragma unroll
                        for (int j = 0; j < kBN / 64; ++j)
                            tma_load_2d(pair ? &tm_b1 : &tm_b0, fb, b_dst + j * kAtomBytes,
                                        c0 + 64 * j, red0);
                    } else {
                        const int red0 = kb * kBR;
                        // A: [64 rows of M] x [128 of N] of dG or dU, MN-major.
#pragma unroll
                        for (int j = 0; j < kBM / 64; ++j)
                            tma_load_2d(second ? &tm_a1 : &tm_a0, fb, a_dst + j * kAtomBytes,
                                        r0 + 64 * j, red0);
                        // B: [64 rows of M] x [BN of K] of X, MN-major.
#pragma unroll
                        for (int j = 0; j < kBN / 64; ++j)
                            tma_load_2d(&tm_b0, fb, b_dst + j * kAtomBytes, c0 + 64 * j, red0);
                    }
                    ++issued;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < C::kStages; ++s) {
                if (issued > s) {
                    const long long uses = (issued - 1 - s) / C::kStages + 1;
                    mbar_wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = make_idesc(1u, kBM, kBN) | kIdescBMnMajor |
                                       (kMode == kModeDw ? kIdescAMnMajor : 0u);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = blockIdx.x; t < num_tiles && !failed; t += gridDim.x) {
                if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sa + stage * kABytes;
                    const uint64_t adesc = kMode == kModeDx
                                               ? sw128_kmajor_desc(a_addr)
                                               : sw128_mnmajor_desc(a_addr, kAtomBytes);
                    const uint64_t bdesc = sw128_mnmajor_desc(sb + stage * C::kBBytes, kAtomBytes);
#pragma unroll
                    for (int kk = 0; kk < kBR / kUmmaK; ++kk) {
                        // K-major: +32 B along the swizzled row (+2); MN-major:
                        // +16 rows of 128 B (+128).
                        const uint64_t a_step = kMode == kModeDx ? 2u * kk : 128u * kk;
                        mma_f16(d_tmem, adesc + a_step, bdesc + 128u * kk, idesc,
                                (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_empty + 8 * stage);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (failed) break;
                mma_commit(bar_tfull + 8 * acc);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            mma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0);
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int quad = warp & 3;
        const uint32_t row_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t buf = se + static_cast<uint32_t>(warp - 2) * kEpiBufBytes;
        const uint32_t swz = static_cast<uint32_t>(lane & 7);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            int mt, nt;
            tile_coords(t, geo.num_m, geo.num_n, mt, nt);
            const int second = (kMode == kModeDw && mt >= geo.row_tiles) ? 1 : 0;
            const int r0 = (mt - second * geo.row_tiles) * kBM;
            const int c0 = nt * kBN;
            if (!mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem_base + row_off + static_cast<uint32_t>(acc * kBN);
#pragma unroll 1
            for (int c = 0; c < kBN / 64; ++c) {
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
                uint32_t v0[32], v1[32];
                tmem_ld_32x32b_x32(tacc + static_cast<uint32_t>(c * 64), v0);
                tmem_ld_32x32b_x32(tacc + static_cast<uint32_t>(c * 64 + 32), v1);
                tmem_ld_wait(v0);
                tmem_ld_wait(v1);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t *src = j < 4 ? v0 : v1;
                    const int e = 8 * (j & 3);
                    uint4 v;
                    v.x = pack_bf16x2(src[e + 0], src[e + 1]);
                    v.y = pack_bf16x2(src[e + 2], src[e + 3]);
                    v.z = pack_bf16x2(src[e + 4], src[e + 5]);
                    v.w = pack_bf16x2(src[e + 6], src[e + 7]);
                    sts_v4(buf + static_cast<uint32_t>(lane) * 128u +
                               ((static_cast<uint32_t>(j) ^ swz) << 4),
                           v);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int x = c0 + c * 64;
                    const int y = r0 + quad * 32;
                    if (x < geo.cols && y < geo.rows) {
                        tma_store_2d(second ? &tm_o1 : &tm_o0, buf, x, y);
                        bulk_commit();
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty + 8 * acc);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait<0>();
    }

    if (failed) atomicOr(&g_gemm_bwd_status, 1u);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

std::atomic<unsigned> g_attr_set_mask[6];

template <int kMode, int kBN>
cudaError_t launch_tiles(const CUtensorMap (&tm)[6], const Geo &geo, const DeviceInfo &dev,
                         cudaStream_t stream) {
    auto kernel = swiglu_gemm_bwd_bf16_kernel<kMode, kBN>;
    constexpr int slot = kMode * 3 + kBN / 64 - 2;
    const unsigned bit = 1u << (dev.device & 31);
    if (!(g_attr_set_mask[slot].load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(Cfg<kBN>::kSmemBytes));
        if (e != cudaSuccess) return e;
        g_attr_set_mask[slot].fetch_or(bit);
    }
    const long long tiles = static_cast<long long>(geo.num_m) * geo.num_n;
    const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
    kernel<<<grid, kThreads, Cfg<kBN>::kSmemBytes, stream>>>(tm[0], tm[1], tm[2], tm[3], tm[4],
                                                             tm[5], geo);
    return cudaGetLastError();
}

}  // namespace

int bwd_gemm_tile_n(int row_tiles_total, int cols, int sm_count) {
    // Predicted time of the raster for each tile width: whole waves of
    // ceil(tiles / SMs), each as long as one tile, whose time is its width
    // divided by the MMA efficiency at that N.  Measured on B200: N = 128
    // (8 KB of shared-memory operands per 64 clocks) reaches about 0.69 of
    // the N = 256 rate; N = 192 is taken as 0.97.  Narrow tiles therefore
    // win only where they fill the last wave much better.
    static const int widths[3] = {256, 192, 128};
    static const double eff[3] = {1.0, 0.97, 0.69};
    int best = 256;
    double best_t = 0.0;
    for (int i = 0; i < 3; ++i) {
        const long long tiles =
            static_cast<long long>(row_tiles_total) * ((cols + widths[i] - 1) / widths[i]);
        const long long waves = (tiles + sm_count - 1) / sm_count;
        const double t = static_cast<double>(waves) * widths[i] / eff[i];
        if (i == 0 || t < best_t * 0.98) {
            best = widths[i];
            best_t = t;
        }
    }
    return best;
}

cudaError_t launch_bwd_dx_bf16(const void *dG, const void *dU, const void *Wg, const void *Wu,
                               void *dX, int M, int K, int N, const DeviceInfo &dev,
                               cudaStream_t stream) {
    Geo geo{};
    geo.rows = M;
    geo.cols = K;
    geo.row_tiles = (M + kBM - 1) / kBM;
    geo.num_m = geo.row_tiles;
    geo.kb_pair = (N + kBR - 1) / kBR;
    const int bn = bwd_gemm_tile_n(geo.num_m, K, dev.sm_count);
    geo.num_n = (K + bn - 1) / bn;
    const CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const uint64_t n_bytes = static_cast<uint64_t>(N) * 2, k_bytes = static_cast<uint64_t>(K) * 2;
    CUtensorMap tm[6];
    if (!encode_tmap_2d(&tm[0], dG, bf16, N, M, n_bytes, kBR, kBM, sw) ||
        !encode_tmap_2d(&tm[1], dU, bf16, N, M, n_bytes, kBR, kBM, sw) ||
        !encode_tmap_2d(&tm[2], Wg, bf16, K, N, k_bytes, 64, kBR, sw) ||
        !encode_tmap_2d(&tm[3], Wu, bf16, K, N, k_bytes, 64, kBR, sw) ||
        !encode_tmap_2d(&tm[4], dX, bf16, K, M, k_bytes, 64, 32, sw)) {
        return cudaErrorInvalidValue;
    }
    tm[5] = tm[4];
    switch (bn) {
        case 128: return launch_tiles<kModeDx, 128>(tm, geo, dev, stream);
        case 192: return launch_tiles<kModeDx, 192>(tm, geo, dev, stream);
        default: return launch_tiles<kModeDx, 256>(tm, geo, dev, stream);
    }
}

cudaError_t launch_bwd_dw_bf16(const void *dG, const void *dU, const void *X, void *dWg,
                               void *dWu, int M, int K, int N, const DeviceInfo &dev,
                               cudaStream_t stream) {
    Geo geo{};
    geo.rows = N;
    geo.cols = K;
    geo.row_tiles = (N + kBM - 1) / kBM;
    geo.num_m = 2 * geo.row_tiles;
    geo.kb_pair = (M + kBR - 1) / kBR;
    const int bn = bwd_gemm_tile_n(geo.num_m, K, dev.sm_count);
    geo.num_n = (K + bn - 1) / bn;
    const CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const uint64_t n_bytes = static_cast<uint64_t>(N) * 2, k_bytes = static_cast<uint64_t>(K) * 2;
    CUtensorMap tm[6];
    if (!encode_tmap_2d(&tm[0], dG, bf16, N, M, n_bytes, 64, kBR, sw) ||
        !encode_tmap_2d(&tm[1], dU, bf16, N, M, n_bytes, 64, kBR, sw) ||
        !encode_tmap_2d(&tm[2], X, bf16, K, M, k_bytes, 64, kBR, sw) ||
        !encode_tmap_2d(&tm[4], dWg, bf16, K, N, k_bytes, 64, 32, sw) ||
        !encode_tmap_2d(&tm[5], dWu, bf16, K, N, k_bytes, 64, 32, sw)) {
        return cudaErrorInvalidValue;
    }
    tm[3] = tm[2];
    switch (bn) {
        case 128: return launch_tiles<kModeDw, 128>(tm, geo, dev, stream);
        case 192: return launch_tiles<kModeDw, 192>(tm, geo, dev, stream);
        default: return launch_tiles<kModeDw, 256>(tm, geo, dev, stream);
    }
}

cudaError_t gemm_bwd_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_gemm_bwd_status, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gemm_bwd_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
