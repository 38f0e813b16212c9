// gemm_tf32x3_2sm.cu -- the fp32 (3xTF32) fused SwiGLU dual GEMM with each
// MMA spread over a pair of SMs (tcgen05 cta_group::2), sm_100a.
//
// Same arithmetic as gemm_tf32x3.cu (hi = the raw operand, lo written by the
// split warps, three kind::tf32 MMAs per 8-deep step, 256-deep chunks folded
// with round-to-nearest adds).  What changes is the shape of one MMA: M = 256
// rows over the two CTAs of a cluster, N = 256 (gate 128 | up 128).  Each CTA
// holds its own 128 rows of X and HALF of the weight rows -- the even CTA the
// 128 rows of Wg, the odd one the 128 rows of Wu -- and the tensor cores of
// the pair exchange the halves.  Per SM and per 16-deep stage that is 16 KB
// loaded and split instead of 24 KB, and 48 KB of operand reads from shared
// memory by the MMAs instead of 72 KB, for the same 128 x 256 outputs per SM:
// the single-SM kernel is bound by shared-memory traffic.
//
// Roles (320 threads per CTA, one CTA per SM, clusters of two):
//  * warp 0 lane 0: TMA producer of its own CTA's stages;
//  * warp 1 lane 0 of the even CTA: MMA issuer for the pair (waits until
//    both CTAs' split warps have prepared a stage; its commits arrive on the
//    barriers of both CTAs); warp 1 of both CTAs allocates and frees the
//    pair's TMEM;
//  * warps 2..5: split (each CTA its own stage), then an arrive on the even
//    CTA's "ready" barrier;
//  * warps 6..9: fold every chunk of their CTA's accumulator rows, then an
//    arrive on the even CTA's "chunk empty" barrier; epilogue of their rows.
// Every wait is bounded; the final cluster barrier is reached by every thread
// of both CTAs in all cases.
#include <atomic>

#include "activation.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tf32x3.cuh"
#include "tmap.cuh"

namespace swiglu {

// Status word of this translation unit's kernel (bit 0 = a wait gave up).
__device__ unsigned int g_gemm_tf32x3_2sm_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;
using gemm::tile_coords;

constexpr int kBM = 128;                 // X rows per CTA (256 per pair)
constexpr int kBN = 128;                 // H columns per tile (gate, up each)
constexpr int kBK = 16;                  // fp32 k per stage: one 64-byte row
constexpr int kStages = 6;
constexpr int kUmmaK = 8;                // k per tcgen05.mma, kind::tf32
constexpr int kAccCols = 2 * kBN;        // gate + up columns
constexpr int kTmemCols = 2 * kAccCols;  // chunk accumulator + running sum
constexpr int kChunkKB = 16;             // k-blocks per accumulation chunk
constexpr int kSplitWarps = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * (kSplitWarps + kEpiWarps);  // 320
constexpr int kFirstSplitWarp = 2;
constexpr int kFirstEpiWarp = kFirstSplitWarp + kSplitWarps;   // 6
constexpr int kGroupPairs = gemm::kGroupMForward / 2;          // 256-row tiles per raster group

constexpr uint32_t kABytes = kBM * kBK * 4;            // 8 KB: this CTA's X rows
constexpr uint32_t kBBytes = kBN * kBK * 4;            // 8 KB: this CTA's weight rows
constexpr uint32_t kRawBytes = kABytes + kBBytes;      // 16 KB loaded per stage
constexpr uint32_t kStageBytes = 2 * kRawBytes;        // + lo copies
constexpr uint32_t kEpiBufBytes = 32 * 128;            // 32 rows x 32 fp32
constexpr uint32_t kOffStages = 0;
constexpr uint32_t kOffEpi = kOffStages + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffEpi + kEpiWarps * kEpiBufBytes;
// full, ready, empty per stage; chunk full, chunk empty, drain
constexpr uint32_t kNumBars = 3 * kStages + 3;
constexpr uint32_t kOffTmemPtr = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemPtr + 8;
constexpr uint32_t kSmemUsed = kOffAbort + 8;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;

static_assert(kSmemBytes <= 232448, "exceeds the 227 KB opt-in shared memory");
static_assert(kRawBytes % 1024 == 0, "lo copies must keep the swizzle alignment");

__device__ __forceinline__ float gated_accurate(int which, float alpha, uint32_t gbits,
                                                uint32_t ubits) {
    return act::gated<true>(which, alpha, __uint_as_float(gbits), __uint_as_float(ubits));
}

__global__ void __launch_bounds__(kThreads, 1)
    swiglu_gemm_tf32x3_2sm_kernel(const __grid_constant__ CUtensorMap tm_x,
                                  const __grid_constant__ CUtensorMap tm_wg,
                                  const __grid_constant__ CUtensorMap tm_wu,
                                  const __grid_constant__ CUtensorMap tm_h,
                                  const __grid_constant__ CUtensorMap tm_g,
                                  const __grid_constant__ CUtensorMap tm_u, int M, int N, int K,
                                  int num_m2_tiles, int num_n_tiles, int which_act, float alpha,
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
    const uint32_t rank = cluster_rank();        // 0: the pair's MMA issuer
    const int pair = static_cast<int>(blockIdx.x) / 2;
    const int num_pairs = static_cast<int>(gridDim.x) / 2;
    const int num_tiles = num_m2_tiles * num_n_tiles;
    const int num_kb = (K + kBK - 1) / kBK;
    const int num_chunks = (num_kb + kChunkKB - 1) / kChunkKB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_ready + 8 * s, 2 * kSplitWarps);  // both CTAs' split warps
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_cfull, 1);
        mbar_init(bar_cempty, 2 * kEpiWarps);                // both CTAs' epilogue warps
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(rank == 0 ? &tm_wg : &tm_wu);
        tma_prefetch_desc(&tm_h);
        if (store_gu) {
            tma_prefetch_desc(&tm_g);
            tma_prefetch_desc(&tm_u);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_ptr), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    // both CTAs' barriers initialised and TMEM allocated before any arrive
    // from the other CTA or any MMA of the pair
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_ptr);
    // the even CTA's barriers, as addresses in the cluster window
    const uint32_t ready_r0 = map_to_rank(bar_ready, 0);
    const uint32_t cempty_r0 = map_to_rank(bar_cempty, 0);

    bool failed = false;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const CUtensorMap *tm_w = rank == 0 ? &tm_wg : &tm_wu;
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int t = pair; t < num_tiles && !failed; t += num_pairs) {
                int mt, nt;
                tile_coords<kGroupPairs>(t, num_m2_tiles, num_n_tiles, mt, nt);
                const int m0 = mt * 2 * kBM + static_cast<int>(rank) * kBM, n0 = nt * kBN;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t st = sst + stage * kStageBytes;
                    mbar_arrive_expect_tx(fb, kRawBytes);
                    tma_load_2d(&tm_x, fb, st, kb * kBK, m0);
                    tma_load_2d(tm_w, fb, st + kABytes, kb * kBK, n0);
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
        if (lane == 0 && rank == 0) {
            // ------------------------------------------ MMA issuer (pair)
            constexpr uint32_t idesc = make_idesc(2u, 2 * kBM, 2 * kBN);
            // the odd CTA's barriers, as addresses in the cluster window
            const uint32_t empty_r1 = map_to_rank(bar_empty, 1);
            const uint32_t cfull_r1 = map_to_rank(bar_cfull, 1);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t chunk_phase = 0;
            for (int t = pair; t < num_tiles && !failed; t += num_pairs) {
                for (int q = 0; q < num_chunks && !failed; ++q) {
                    // both CTAs' epilogue warps must have read the previous chunk
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
                            const uint32_t o = 2u * kk;
                            const uint32_t acc = (kb == q * kChunkKB && kk == 0) ? 0u : 1u;
                            mma_tf32_pair(tmem_base, a_lo + o, b_hi + o, idesc, acc);
                            mma_tf32_pair(tmem_base, a_hi + o, b_lo + o, idesc, 1u);
                            mma_tf32_pair(tmem_base, a_hi + o, b_hi + o, idesc, 1u);
                        }
                        // the stage is free in both CTAs
                        mma_commit_pair(bar_empty + 8 * stage);
                        mma_commit_pair(empty_r1 + 8 * stage);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (failed) break;
                    mma_commit_pair(bar_cfull);
                    mma_commit_pair(cfull_r1);
                    chunk_phase ^= 1u;
                }
            }
            mma_commit_pair(bar_drain);
            mbar_wait_drain(bar_drain, 0);
        }
    } else if (warp < kFirstEpiWarp) {
        // ---------------------------------------------------- hi/lo split
        const int sidx = threadIdx.x - 32 * kFirstSplitWarp;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        for (int t = pair; t < num_tiles && !failed; t += num_pairs) {
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                    failed = true;
                    break;
                }
                tf32x3::split_stage<kRawBytes, 32 * kSplitWarps>(sst + stage * kStageBytes, sidx);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(ready_r0 + 8 * stage);
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
        const uint32_t chunk_acc = tmem_base + row_off;
        const uint32_t run_acc = tmem_base + row_off + kAccCols;
        const uint32_t buf = se + static_cast<uint32_t>(warp - kFirstEpiWarp) * kEpiBufBytes;
        const uint32_t swz = static_cast<uint32_t>(lane & 7);
        uint32_t chunk_phase = 0;
        for (int t = pair; t < num_tiles && !failed; t += num_pairs) {
            int mt, nt;
            tile_coords<kGroupPairs>(t, num_m2_tiles, num_n_tiles, mt, nt);
            const int m0 = mt * 2 * kBM + static_cast<int>(rank) * kBM, n0 = nt * kBN;
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
                if (lane == 0) mbar_arrive_remote(cempty_r0);
            }
            if (failed) break;
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
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const int e = 4 * j + e4;
                            pv[e4] = what == 0
                                         ? __float_as_uint(gated_accurate(which_act, alpha, g[e], u[e]))
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

    if (failed) atomicOr(&g_gemm_tf32x3_2sm_status, 1u);

    tc_fence_before();
    __syncthreads();
    // the pair's MMAs have completed (the issuer drained them) and both CTAs'
    // epilogues are done before either frees TMEM or leaves
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

std::atomic<unsigned> g_attr_set_mask{0};

}  // namespace

bool gemm_tf32x3_2sm_worth(int M) { return M > kBM; }

cudaError_t launch_gemm_tf32x3_2sm(const void *X, const void *Wg, const void *Wu, void *H, int M,
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
        cudaError_t e = cudaFuncSetAttribute(swiglu_gemm_tf32x3_2sm_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBytes));
        if (e != cudaSuccess) return e;
        g_attr_set_mask.fetch_or(bit);
    }
    const int num_m2 = (M + 2 * kBM - 1) / (2 * kBM);
    const int num_n = (N + kBN - 1) / kBN;
    const long long tiles = static_cast<long long>(num_m2) * num_n;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // as many pairs as can be resident at once (persistent grid)
    int max_clusters = 0;
    cfg.gridDim = dim3(2);
    cudaError_t e = cudaOccupancyMaxActiveClusters(&max_clusters, swiglu_gemm_tf32x3_2sm_kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (max_clusters < 1) return cudaErrorInvalidConfiguration;
    const long long pairs = tiles < max_clusters ? tiles : max_clusters;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    e = cudaLaunchKernelEx(&cfg, swiglu_gemm_tf32x3_2sm_kernel, tx, twg, twu, th, tg, tu, M, N, K,
                           num_m2, num_n, epi.activation, epi.gate_multiplier, store_gu ? 1 : 0);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t gemm_tf32x3_2sm_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_gemm_tf32x3_2sm_status,
                                              sizeof(unsigned int), 0, cudaMemcpyDeviceToHost,
                                              stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gemm_tf32x3_2sm_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
