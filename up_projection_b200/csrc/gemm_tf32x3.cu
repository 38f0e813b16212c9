// gemm_tf32x3.cu -- fused SwiGLU dual GEMM for fp32 inputs, near-IEEE
// accuracy on the tensor cores by 3xTF32 splitting, sm_100a.
//
// Why: Liger-Kernel issue #1383 ("[RFC] Testing Methodology for FP32
// Convergence Tests ...", Root Cause) shows a fused gate/up kernel whose fp32
// matmuls ran on the TF32 tensor-core path failing fp32 parity, while forcing
// IEEE FMA overflowed shared memory.  Here every fp32 operand is split
//     a = hi + lo,   hi = trunc_tf32(a),   lo = rna_tf32(a - hi)
// and each product is formed as hi*hi + hi*lo + lo*hi (the lo*lo term, below
// 2^-22 relative, is dropped), all accumulated in fp32 in tensor memory.
// This is the split-precision refinement of Markidis et al. (2018, "NVIDIA
// Tensor Core Programmability, Performance & Precision") in the error-
// corrected TF32 form of Ootomo & Yokota (2022, "Recovering single precision
// accuracy from Tensor Cores while surpassing the FP32 theoretical peak
// performance"), written here from the mathematics.
//
// Structure (one CTA per SM, persistent over 128 x 128 output tiles):
//  * warp 0 (one thread): TMA producer -- raw fp32 X [128 x 16] and the
//    stacked [Wg; Wu] tile [256 x 16] per 16-deep k-block, 64-byte swizzle,
//    into a 4-stage ring;
//  * warps 2..5: split -- each raw stage serves as hi as it landed (the MMA
//    reads the top 19 bits of each element: trunc_tf32) and lo is written to
//    a parallel buffer with the same (swizzled) layout;
//  * warp 1 (one thread): MMA issuer -- per 8-deep step three
//    tcgen05.mma kind::tf32 (M=128, N=256): Xhi*[Wg;Wu]hi, Xhi*[Wg;Wu]lo,
//    Xlo*[Wg;Wu]hi into the chunk accumulator (gate columns 0..127, up
//    columns 128..255);
//  * warps 6..9: accumulation and epilogue.  The tensor cores' fp32
//    accumulation loses up to about one unit in the last place of the running
//    sum per accumulate step, an error that grows linearly with K.  So each
//    tile's K range is cut into chunks of kChunkKB k-blocks (256 k): the MMAs
//    of a chunk start from zero in the chunk accumulator (TMEM columns 0..255)
//    and these warps fold every finished chunk into a running sum (TMEM
//    columns 256..511) with round-to-nearest fp32 adds on the CUDA cores,
//    releasing the chunk accumulator right after reading it.  After the last
//    chunk: h = g * sigmoid(g) * u in fp32 with expf and IEEE division, staged
//    (128-byte swizzle) and stored by TMA while the next tile's MMAs run.
// All waits are bounded as in the bf16 kernel.
#include <atomic>

#include "activation.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tf32x3.cuh"
#include "tmap.cuh"

namespace swiglu {

// Status word of this translation unit's kernel (bit 0 = a wait gave up).
__device__ unsigned int g_gemm_tf32x3_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;
using gemm::tile_coords;

constexpr int kBM = 128;
constexpr int kBN = 128;                 // H columns per tile (gate, up each)
constexpr int kBK = 16;                  // fp32 k per stage: one 64-byte row
constexpr int kStages = 4;
constexpr int kUmmaK = 8;                // k per tcgen05.mma, kind::tf32
constexpr int kAccCols = 2 * kBN;        // gate + up columns
constexpr int kTmemCols = 2 * kAccCols;  // chunk accumulator + running sum
constexpr int kChunkKB = 16;             // k-blocks per accumulation chunk
constexpr int kSplitWarps = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * (kSplitWarps + kEpiWarps);  // 320
constexpr int kFirstSplitWarp = 2;
constexpr int kFirstEpiWarp = kFirstSplitWarp + kSplitWarps;   // 6

constexpr uint32_t kABytes = kBM * kBK * 4;            // 8 KB
constexpr uint32_t kBBytes = 2 * kBN * kBK * 4;        // 16 KB: Wg rows, Wu rows
constexpr uint32_t kRawBytes = kABytes + kBBytes;      // 24 KB loaded per stage
constexpr uint32_t kStageBytes = 2 * kRawBytes;        // + lo copies
constexpr uint32_t kEpiBufBytes = 32 * 128;            // 32 rows x 32 fp32
// Per stage: [A hi | B hi | A lo | B lo]; the hi half is what TMA loads.
constexpr uint32_t kOffStages = 0;
constexpr uint32_t kOffEpi = kOffStages + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffEpi + kEpiWarps * kEpiBufBytes;
constexpr uint32_t kNumBars = 3 * kStages + 3;  // full, ready, empty, chunk_full, chunk_empty, drain
constexpr uint32_t kOffTmemPtr = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemPtr + 8;
constexpr uint32_t kSmemUsed = kOffAbort + 8;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;

static_assert(kSmemBytes <= 232448, "exceeds the 227 KB opt-in shared memory");
static_assert(kRawBytes % 1024 == 0, "lo copies must keep the swizzle alignment");

// h = act(alpha g) * u in fp32 with expf / tanhf and IEEE division (a few
// ulp in total).
__device__ __forceinline__ float gated_accurate(int which, float alpha, uint32_t gbits,
                                                uint32_t ubits) {
    return act::gated<true>(which, alpha, __uint_as_float(gbits), __uint_as_float(ubits));
}

__global__ void __launch_bounds__(kThreads, 1)
    swiglu_gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tm_x,
                              const __grid_constant__ CUtensorMap tm_wg,
                              const __grid_constant__ CUtensorMap tm_wu,
                              const __grid_constant__ CUtensorMap tm_h,
                              const __grid_constant__ CUtensorMap tm_g,
                              const __grid_constant__ CUtensorMap tm_u, int M, int N, int K,
                              int num_m_tiles, int num_n_tiles, int which_act, float alpha,
                              int store_gu) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const uint32_t sst = base + kOffStages;
    const uint32_t se = base + kOffEpi;
    const uint32_t bar_full = base + kOffBar;
    const uint32_t bar_ready = bar_full + 8 * kStages;
    const uint32_t bar_empty = bar_ready + 8 * kStages;
    const uint32_t bar_cfull = bar_empty + 8 * kStages;
    const uint32_t bar_cempty = bar_cfull + 8;
    const uint32_t bar_drain = bar_cempty + 8;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(gbase + kOffTmemPtr);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + kOffAbort);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int num_tiles = num_m_tiles * num_n_tiles;
    const int num_kb = (K + kBK - 1) / kBK;
    const int num_chunks = (num_kb + kChunkKB - 1) / kChunkKB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_ready + 8 * s, kSplitWarps);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_cfull, 1);
        mbar_init(bar_cempty, kEpiWarps);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_wg);
        tma_prefetch_desc(&tm_wu);
        tma_prefetch_desc(&tm_h);
        if (store_gu) {
            tma_prefetch_desc(&tm_g);
            tma_prefetch_desc(&tm_u);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), kTmemCols);
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
                tile_coords<gemm::kGroupMForward>(t, num_m_tiles, num_n_tiles, mt, nt);
                const int m0 = mt * kBM, n0 = nt * kBN;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t st = sst + stage * kStageBytes;
                    mbar_arrive_expect_tx(fb, kRawBytes);
                    tma_load_2d(&tm_x, fb, st, kb * kBK, m0);
                    tma_load_2d(&tm_wg, fb, st + kABytes, kb * kBK, n0);
                    tma_load_2d(&tm_wu, fb, st + kABytes + kBBytes / 2, kb * kBK, n0);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < kStages; ++s) {
                if (issued > s) {
                    const long long uses = (issued - 1 - s) / kStages + 1;
                    mbar_wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = make_idesc(2u, kBM, 2 * kBN);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t chunk_phase = 0;  // parity of the chunk accumulator's uses
            for (int t = blockIdx.x; t < num_tiles && !failed; t += gridDim.x) {
                for (int q = 0; q < num_chunks && !failed; ++q) {
                    // the epilogue warps must have read the previous chunk
                    if (!mbar_wait(bar_cempty, chunk_phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const int kb_end = min(num_kb, (q + 1) * kChunkKB);
                    for (int kb = q * kChunkKB; kb < kb_end; ++kb) {
                        if (!mbar_wait(bar_ready + 8 * stage, phase, abort_flag)) {
                            failed = true;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t st = sst + stage * kStageBytes;
                        const uint64_t a_hi = sw64_kmajor_desc(st);
                        const uint64_t b_hi = sw64_kmajor_desc(st + kABytes);
                        const uint64_t a_lo = sw64_kmajor_desc(st + kRawBytes);
                        const uint64_t b_lo = sw64_kmajor_desc(st + kRawBytes + kABytes);
#pragma unroll
                        for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                            // +32 bytes along K inside the 64-byte swizzled row.
                            const uint32_t o = 2u * kk;
                            const uint32_t acc = (kb == q * kChunkKB && kk == 0) ? 0u : 1u;
                            mma_tf32(tmem_base, a_lo + o, b_hi + o, idesc, acc);
                            mma_tf32(tmem_base, a_hi + o, b_lo + o, idesc, 1u);
                            mma_tf32(tmem_base, a_hi + o, b_hi + o, idesc, 1u);
                        }
                        mma_commit(bar_empty + 8 * stage);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (failed) break;
                    mma_commit(bar_cfull);
                    chunk_phase ^= 1u;
                }
            }
            mma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0);
        }
    } else if (warp < kFirstEpiWarp) {
        // ---------------------------------------------------- hi/lo split
        const int sidx = threadIdx.x - 32 * kFirstSplitWarp;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        for (int t = blockIdx.x; t < num_tiles && !failed; t += gridDim.x) {
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                    failed = true;
                    break;
                }
                tf32x3::split_stage<kRawBytes, 32 * kSplitWarps>(sst + stage * kStageBytes, sidx);
                // make the generic-proxy writes visible to the tensor cores
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_ready + 8 * stage);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------ accumulation + epilogue
        const int quad = warp & 3;
        const uint32_t row_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t chunk_acc = tmem_base + row_off;             // cols 0..255
        const uint32_t run_acc = tmem_base + row_off + kAccCols;    // cols 256..511
        const uint32_t buf = se + static_cast<uint32_t>(warp - kFirstEpiWarp) * kEpiBufBytes;
        const uint32_t swz = static_cast<uint32_t>(lane & 7);
        uint32_t chunk_phase = 0;
        for (int t = blockIdx.x; t < num_tiles && !failed; t += gridDim.x) {
            int mt, nt;
            tile_coords<gemm::kGroupMForward>(t, num_m_tiles, num_n_tiles, mt, nt);
            const int m0 = mt * kBM, n0 = nt * kBN;
            // fold every chunk into the running sum and release the chunk
            // accumulator; the next tile's first chunk then overlaps the
            // output below
            for (int q = 0; q < num_chunks; ++q) {
                if (!mbar_wait(bar_cfull, chunk_phase, abort_flag)) {
                    failed = true;
                    break;
                }
                chunk_phase ^= 1u;
                tc_fence_after();
                tf32x3::fold_chunk<kAccCols>(chunk_acc, run_acc, q);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_cempty);
            }
            if (failed) break;
            // output from the running sum: H = act(alpha g) u, then (training
            // forward) G and U themselves
            const int outputs = store_gu ? 3 : 1;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
#pragma unroll 1
                for (int what = 0; what < outputs; ++what) {
                    if (lane == 0) bulk_wait_read<0>();
                    __syncwarp();
                    uint32_t g[32], u[32];
                    if (what != 2) tmem_ld_32x32b_x32(run_acc + 32u * c, g);
                    if (what != 1) tmem_ld_32x32b_x32(run_acc + kBN + 32u * c, u);
                    tmem_ld_wait(g);
                    tmem_ld_wait(u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint4 v;
                        uint32_t *pv = &v.x;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int e = 4 * j + q;
                            pv[q] = what == 0 ? __float_as_uint(gated_accurate(which_act, alpha, g[e], u[e]))
                                              : (what == 1 ? g[e] : u[e]);
                        }
                        sts_v4(buf + static_cast<uint32_t>(lane) * 128u +
                                   ((static_cast<uint32_t>(j) ^ swz) << 4),
                               v);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int x = n0 + c * 32;
                        const int y = m0 + quad * 32;
                        if (x < N && y < M) {
                            const CUtensorMap *dst = what == 0 ? &tm_h : (what == 1 ? &tm_g : &tm_u);
                            tma_store_2d(dst, buf, x, y);
                            bulk_commit();
                        }
                    }
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
    }

    if (failed) atomicOr(&g_gemm_tf32x3_status, 1u);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

std::atomic<unsigned> g_attr_set_mask{0};

}  // namespace

cudaError_t launch_gemm_tf32x3(const void *X, const void *Wg, const void *Wu, void *H, int M,
                               int K, int N, const Epilogue &epi, const DeviceInfo &dev,
                               cudaStream_t stream) {
    CUtensorMap tx, twg, twu, th, tg, tu;
    const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const CUtensorMapSwizzle sw64 = CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapSwizzle sw128 = CU_TENSOR_MAP_SWIZZLE_128B;
    const bool store_gu = epi.G != nullptr;
    const uint64_t hrow = static_cast<uint64_t>(N) * 4;
    if (!encode_tmap_2d(&tx, X, f32, K, M, static_cast<uint64_t>(K) * 4, kBK, kBM, sw64) ||
        !encode_tmap_2d(&twg, Wg, f32, K, N, static_cast<uint64_t>(K) * 4, kBK, kBN, sw64) ||
        !encode_tmap_2d(&twu, Wu, f32, K, N, static_cast<uint64_t>(K) * 4, kBK, kBN, sw64) ||
        !encode_tmap_2d(&th, H, f32, N, M, hrow, 32, 32, sw128) ||
        !encode_tmap_2d(&tg, store_gu ? epi.G : H, f32, N, M, hrow, 32, 32, sw128) ||
        !encode_tmap_2d(&tu, store_gu ? epi.U : H, f32, N, M, hrow, 32, 32, sw128)) {
        return cudaErrorInvalidValue;
    }
    const unsigned bit = 1u << (dev.device & 31);
    if (!(g_attr_set_mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(swiglu_gemm_tf32x3_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBytes));
        if (e != cudaSuccess) return e;
        g_attr_set_mask.fetch_or(bit);
    }
    const int num_m = (M + kBM - 1) / kBM;
    const int num_n = (N + kBN - 1) / kBN;
    const long long tiles = static_cast<long long>(num_m) * num_n;
    const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
    swiglu_gemm_tf32x3_kernel<<<grid, kThreads, kSmemBytes, stream>>>(
        tx, twg, twu, th, tg, tu, M, N, K, num_m, num_n, epi.activation, epi.gate_multiplier,
        store_gu ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t gemm_tf32x3_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_gemm_tf32x3_status,
                                              sizeof(unsigned int), 0, cudaMemcpyDeviceToHost,
                                              stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gemm_tf32x3_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
