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
// Pair form (output tiles of 256 rows, where there is more than one 128-row
// block): each MMA covers the 256 rows over the two CTAs of a cluster
// (tcgen05 cta_group::2); a CTA loads its own 128 rows of A and half of the
// tile's B columns, so its shared-memory operand traffic per MFLOP falls by a
// third.  Both CTAs' copies are counted on the even CTA's full barrier, whose
// MMA-issuing thread commits every stage and accumulator to both CTAs.
//
// One launch can run dX, dW or both, on the static schedule of
// gemm_common.cuh (each CTA: its dX tiles first, then dW tiles in the order
// the CTAs free up), so the combined call ends in one balanced tail.
//
// MN-major tiles are TMA boxes {64, 64} in the 128-byte swizzle, one per
// 64-wide MN atom; the UMMA descriptor walks atoms with its leading byte
// offset (ptx.cuh).  Out-of-range rows/columns/reduction steps are
// zero-filled by TMA on load and clipped on store, so any M, N, K that are
// multiples of 8 (16-byte rows) work, with ragged tails.  Every wait is
// bounded: a stuck pipeline sets the status word and the kernel returns
// after releasing what it holds.
#include <cuda_bf16.h>

#include <string.h>

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

constexpr int kBM = 128;             // output rows per tile (= MMA M)
constexpr int kBR = 64;              // reduction depth per stage (128-byte rows)
constexpr int kUmmaK = 16;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kAtomBytes = 64 * kBR * 2;   // MN-major atom: 64 x 64 bf16 = 8 KB
constexpr uint32_t kABytes = kBM * kBR * 2;     // 16 KB either way
constexpr uint32_t kEpiBufBytes = 32 * 128;     // 32 rows x 64 bf16
constexpr uint32_t kRingBudget = 200 * 1024;

template <int kBN, bool kPair>
struct Cfg {
    static constexpr int kRows = kPair ? 2 * kBM : kBM;     // output rows per tile
    static constexpr int kBCols = kPair ? kBN / 2 : kBN;    // B columns this CTA loads
    static constexpr uint32_t kBBytes = kBCols * kBR * 2;
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
    static_assert(kBCols % 64 == 0, "whole 64-wide atoms in each CTA of a pair");
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB opt-in shared memory");
};

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<uint32_t *>(&v);
}

// Geometry of the two tile kinds and the schedule of one launch.
struct Plan {
    int M, N, K;
    int dx_num_m, dw_row_tiles, dw_num_m, num_n;   // tiles: dx_num_m x num_n, dw_num_m x num_n
    int dx_kb, dw_kb;                              // 64-deep reduction blocks per tile
    int kb_pair;                                   // dX: blocks of one pair (dG Wg, dU Wu)
    gemm::BwdSched sched;
};

// Tensor maps of both kinds (only those of the kinds a launch runs are used).
struct Maps {
    CUtensorMap dx_a[2];   // dG, dU: K-major {64, 128}
    CUtensorMap dx_b[2];   // Wg, Wu: MN-major atoms {64, 64}
    CUtensorMap dx_o;      // dX
    CUtensorMap dw_a[2];   // dG, dU: MN-major atoms {64, 64}
    CUtensorMap dw_b;      // X: MN-major atoms {64, 64}
    CUtensorMap dw_o[2];   // dWg, dWu
};

struct TileInfo {
    int kind, r0, c0, num_kb, second;
};

// The seq-th tile of unit `unit` of `units` (a CTA, or a pair of CTAs of
// which this is number `rank`); r0 is this CTA's first output row.
template <int kBN, bool kPair>
__device__ __forceinline__ bool next_tile(const Plan &p, int seq, TileInfo &ti, int unit,
                                          int units, int rank) {
    constexpr int kRows = Cfg<kBN, kPair>::kRows;
    int kind, t;
    if (!gemm::bwd_tile_of(p.sched, unit, units, seq, kind, t)) return false;
    int mt, nt;
    ti.kind = kind;
    if (kind == gemm::kTileDx) {
        tile_coords<gemm::kGroupMBackward>(t, p.dx_num_m, p.num_n, mt, nt);
        ti.second = 0;
        ti.r0 = mt * kRows + rank * kBM;
        ti.num_kb = p.dx_kb;
    } else {
        tile_coords<gemm::kGroupMBackward>(t, p.dw_num_m, p.num_n, mt, nt);
        ti.second = mt >= p.dw_row_tiles ? 1 : 0;
        ti.r0 = (mt - ti.second * p.dw_row_tiles) * kRows + rank * kBM;
        ti.num_kb = p.dw_kb;
    }
    ti.c0 = nt * kBN;
    return true;
}

// TMA load of one box; in the pair form its completion is counted on the
// even CTA's barrier (`bar`: its cluster address).
template <bool kPair>
__device__ __forceinline__ void load_box(const CUtensorMap *map, uint32_t bar, uint32_t dst,
                                         int32_t x, int32_t y) {
    if constexpr (kPair)
        tma_load_2d_pair(map, bar, dst, x, y);
    else
        tma_load_2d(map, bar, dst, x, y);
}

template <int kBN, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
    swiglu_gemm_bwd_bf16_kernel(const __grid_constant__ Maps maps, const Plan plan) {
    using C = Cfg<kBN, kPair>;
    constexpr int kBCols = C::kBCols;
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
    // kPair: CTA `rank` of pair `unit`; rank 0 issues the pair's MMAs
    const int rank = kPair ? static_cast<int>(cluster_rank()) : 0;
    const int unit = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
    const int units = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
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
        if (plan.sched.T_dx > 0) {
            tma_prefetch_desc(&maps.dx_a[0]);
            tma_prefetch_desc(&maps.dx_a[1]);
            tma_prefetch_desc(&maps.dx_b[0]);
            tma_prefetch_desc(&maps.dx_b[1]);
            tma_prefetch_desc(&maps.dx_o);
        }
        if (plan.sched.T_dw > 0) {
            tma_prefetch_desc(&maps.dw_a[0]);
            tma_prefetch_desc(&maps.dw_a[1]);
            tma_prefetch_desc(&maps.dw_b);
            tma_prefetch_desc(&maps.dw_o[0]);
            tma_prefetch_desc(&maps.dw_o[1]);
        }
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(smem_u32(tmem_ptr), C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_ptr), C::kTmemCols);
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
    TileInfo ti;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            // kPair: every copy of both CTAs is counted on the even CTA's
            // full barrier, whose producer expects the pair's bytes
            const uint32_t full_r0 = kPair ? map_to_rank(bar_full, 0) : 0u;
            // this CTA's first B column within the tile
            const int bc = rank * kBCols;
            for (int seq = 0; !failed && next_tile<kBN, kPair>(plan, seq, ti, unit, units, rank);
                 ++seq) {
                for (int kb = 0; kb < ti.num_kb; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t a_dst = sa + stage * kABytes;
                    const uint32_t b_dst = sb + stage * C::kBBytes;
                    uint32_t fb = bar_full + 8 * stage;
                    if constexpr (kPair) {
                        if (rank == 0) mbar_arrive_expect_tx(fb, 2 * C::kStageBytes);
                        fb = full_r0 + 8 * stage;
                    } else {
                        mbar_arrive_expect_tx(fb, C::kStageBytes);
                    }
                    if (ti.kind == gemm::kTileDx) {
                        const int pair = kb >= plan.kb_pair ? 1 : 0;
                        const int red0 = (kb - pair * plan.kb_pair) * kBR;
                        // A: [128 rows of dG or dU] x [64 of N], K-major.
                        load_box<kPair>(&maps.dx_a[pair], fb, a_dst, red0, ti.r0);
                        // B: [64 rows of Wg or Wu] x [this CTA's columns of K],
                        // MN-major atoms.
#pragma unroll
                        for (int j = 0; j < kBCols / 64; ++j)
                            load_box<kPair>(&maps.dx_b[pair], fb, b_dst + j * kAtomBytes,
                                            ti.c0 + bc + 64 * j, red0);
                    } else {
                        const int red0 = kb * kBR;
                        // A: [64 rows of M] x [128 of N] of dG or dU, MN-major.
#pragma unroll
                        for (int j = 0; j < kBM / 64; ++j)
                            load_box<kPair>(&maps.dw_a[ti.second], fb, a_dst + j * kAtomBytes,
                                            ti.r0 + 64 * j, red0);
                        // B: [64 rows of M] x [this CTA's columns of K] of X,
                        // MN-major.
#pragma unroll
                        for (int j = 0; j < kBCols / 64; ++j)
                            load_box<kPair>(&maps.dw_b, fb, b_dst + j * kAtomBytes,
                                            ti.c0 + bc + 64 * j, red0);
                    }
                    ++issued;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Never leave while a load issued here may still write shared
            // memory.  (kPair: the even CTA's full barriers count the copies
            // of both CTAs; the odd CTA's copies are consumed by the pair's
            // MMAs before the final cluster barrier.)
            for (int s = 0; s < C::kStages && (!kPair || rank == 0); ++s) {
                if (issued > s) {
                    const long long uses = (issued - 1 - s) / C::kStages + 1;
                    mbar_wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_dx = make_idesc(1u, C::kRows, kBN) | kIdescBMnMajor;
            constexpr uint32_t idesc_dw = idesc_dx | kIdescAMnMajor;
            // kPair: the odd CTA's barriers, as addresses in the cluster window
            const uint32_t empty_r1 = kPair ? map_to_rank(bar_empty, 1) : 0u;
            const uint32_t tfull_r1 = kPair ? map_to_rank(bar_tfull, 1) : 0u;
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int seq = 0; !failed && next_tile<kBN, kPair>(plan, seq, ti, unit, units, rank);
                 ++seq) {
                const bool dx = ti.kind == gemm::kTileDx;
                const uint32_t idesc = dx ? idesc_dx : idesc_dw;
                if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, abort_flag)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
                for (int kb = 0; kb < ti.num_kb; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sa + stage * kABytes;
                    const uint64_t adesc = dx ? sw128_kmajor_desc(a_addr)
                                              : sw128_mnmajor_desc(a_addr, kAtomBytes);
                    const uint64_t bdesc = sw128_mnmajor_desc(sb + stage * C::kBBytes, kAtomBytes);
#pragma unroll
                    for (int kk = 0; kk < kBR / kUmmaK; ++kk) {
                        // K-major: +32 B along the swizzled row (+2); MN-major:
                        // +16 rows of 128 B (+128).
                        const uint64_t a_step = dx ? 2u * kk : 128u * kk;
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        if constexpr (kPair)
                            mma_f16_pair(d_tmem, adesc + a_step, bdesc + 128u * kk, idesc, accum);
                        else
                            mma_f16(d_tmem, adesc + a_step, bdesc + 128u * kk, idesc, accum);
                    }
                    if constexpr (kPair) {
                        // the stage is free in both CTAs
                        mma_commit_pair(bar_empty + 8 * stage);
                        mma_commit_pair(empty_r1 + 8 * stage);
                    } else {
                        mma_commit(bar_empty + 8 * stage);
                    }
                    if (++stage == C::kStages) {
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
        const int quad = warp & 3;
        const uint32_t row_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t buf = se + static_cast<uint32_t>(warp - 2) * kEpiBufBytes;
        const uint32_t swz = static_cast<uint32_t>(lane & 7);
        // kPair: the accumulator is released on the even CTA's barrier
        const uint32_t tempty_r0 = kPair ? map_to_rank(bar_tempty, 0) : 0u;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int seq = 0; next_tile<kBN, kPair>(plan, seq, ti, unit, units, rank); ++seq) {
            if (!mbar_wait(bar_tfull + 8 * acc, acc_phase, abort_flag)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const bool dx = ti.kind == gemm::kTileDx;
            const CUtensorMap *out = dx ? &maps.dx_o : &maps.dw_o[ti.second];
            const int rows = dx ? plan.M : plan.N;
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
                    const int x = ti.c0 + c * 64;
                    const int y = ti.r0 + quad * 32;
                    if (x < plan.K && y < rows) {
                        tma_store_2d(out, buf, x, y);
                        bulk_commit();
                    }
                }
            }
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

    if (failed) atomicOr(&g_gemm_bwd_status, 1u);

    tc_fence_before();
    __syncthreads();
    // kPair: the pair's MMAs have completed (the issuer drained them) and
    // both epilogues are done before either CTA frees TMEM or leaves
    if constexpr (kPair) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        __syncwarp();
        if constexpr (kPair)
            tmem_dealloc_pair(tmem_base, C::kTmemCols);
        else
            tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// Bit (device & 31) set once the kernel's shared-memory attribute is set on
// that device; one mask per (width, form).
std::atomic<unsigned> g_attr_set_mask[6];

template <int kBN, bool kPair>
cudaError_t set_smem_attr(const DeviceInfo &dev) {
    constexpr int slot = (kBN / 64 - 2) + (kPair ? 3 : 0);
    const unsigned bit = 1u << (dev.device & 31);
    if (!(g_attr_set_mask[slot].load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(swiglu_gemm_bwd_bf16_kernel<kBN, kPair>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(Cfg<kBN, kPair>::kSmemBytes));
        if (e != cudaSuccess) return e;
        g_attr_set_mask[slot].fetch_or(bit);
    }
    return cudaSuccess;
}

void set_cluster_attr(cudaLaunchAttribute &a) {
    a.id = cudaLaunchAttributeClusterDimension;
    a.val.clusterDim.x = 2;
    a.val.clusterDim.y = 1;
    a.val.clusterDim.z = 1;
}

// `units`: CTAs, or pairs of CTAs (kPair: a cluster of two per pair).
template <int kBN, bool kPair>
cudaError_t launch_width(const Maps &maps, const Plan &plan, int units, const DeviceInfo &dev,
                         cudaStream_t stream) {
    cudaError_t e = set_smem_attr<kBN, kPair>(dev);
    if (e != cudaSuccess) return e;
    if constexpr (kPair) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(2 * units));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = Cfg<kBN, kPair>::kSmemBytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        set_cluster_attr(attr[0]);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, swiglu_gemm_bwd_bf16_kernel<kBN, kPair>, maps, plan);
        if (e != cudaSuccess) return e;
    } else {
        swiglu_gemm_bwd_bf16_kernel<kBN, kPair>
            <<<units, kThreads, Cfg<kBN, kPair>::kSmemBytes, stream>>>(maps, plan);
    }
    return cudaGetLastError();
}

std::atomic<int> g_pair_units[64];

// Pairs of SMs that can run the pair form at once on this device (cached;
// 0 where it cannot run).  One CTA per SM in every form, so the count does
// not depend on the tile width.
int pair_units(const DeviceInfo &dev) {
    if (dev.device < 0 || dev.device >= 64) return 0;
    int u = g_pair_units[dev.device].load();
    if (u != 0) return u > 0 ? u : 0;
    u = -1;
    if (set_smem_attr<256, true>(dev) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = Cfg<256, true>::kSmemBytes;
        cudaLaunchAttribute attr[1];
        set_cluster_attr(attr[0]);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, swiglu_gemm_bwd_bf16_kernel<256, true>, &cfg) ==
                cudaSuccess && n > 0)
            u = n;
        else
            (void)cudaGetLastError();
    }
    g_pair_units[dev.device].store(u);
    return u > 0 ? u : 0;
}

// Encodes the maps of the kinds requested and launches one persistent grid
// over all their tiles, `bn` columns wide; pair: the pair form (256-row
// tiles, a pair of SMs per tile; bn 128 or 256).
cudaError_t launch_plan(const void *dG, const void *dU, const void *Wg, const void *Wu,
                        const void *X, void *dX, void *dWg, void *dWu, int M, int K, int N,
                        bool do_dx, bool do_dw, int bn, bool pair, const DeviceInfo &dev,
                        cudaStream_t stream) {
    const CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const uint64_t n_bytes = static_cast<uint64_t>(N) * 2, k_bytes = static_cast<uint64_t>(K) * 2;
    Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (do_dx &&
        (!encode_tmap_2d(&maps.dx_a[0], dG, bf16, N, M, n_bytes, kBR, kBM, sw) ||
         !encode_tmap_2d(&maps.dx_a[1], dU, bf16, N, M, n_bytes, kBR, kBM, sw) ||
         !encode_tmap_2d(&maps.dx_b[0], Wg, bf16, K, N, k_bytes, 64, kBR, sw) ||
         !encode_tmap_2d(&maps.dx_b[1], Wu, bf16, K, N, k_bytes, 64, kBR, sw) ||
         !encode_tmap_2d(&maps.dx_o, dX, bf16, K, M, k_bytes, 64, 32, sw)))
        return cudaErrorInvalidValue;
    if (do_dw &&
        (!encode_tmap_2d(&maps.dw_a[0], dG, bf16, N, M, n_bytes, 64, kBR, sw) ||
         !encode_tmap_2d(&maps.dw_a[1], dU, bf16, N, M, n_bytes, 64, kBR, sw) ||
         !encode_tmap_2d(&maps.dw_b, X, bf16, K, M, k_bytes, 64, kBR, sw) ||
         !encode_tmap_2d(&maps.dw_o[0], dWg, bf16, K, N, k_bytes, 64, 32, sw) ||
         !encode_tmap_2d(&maps.dw_o[1], dWu, bf16, K, N, k_bytes, 64, 32, sw)))
        return cudaErrorInvalidValue;
    if (pair && bn == 192) bn = 256;   // a pair splits the width into whole 64-wide atoms
    const int rows = pair ? 2 * kBM : kBM;
    Plan plan{};
    plan.M = M;
    plan.N = N;
    plan.K = K;
    plan.num_n = (K + bn - 1) / bn;
    plan.dx_num_m = (M + rows - 1) / rows;
    plan.dw_row_tiles = (N + rows - 1) / rows;
    plan.dw_num_m = 2 * plan.dw_row_tiles;
    plan.kb_pair = (N + kBR - 1) / kBR;
    plan.dx_kb = 2 * plan.kb_pair;
    plan.dw_kb = (M + kBR - 1) / kBR;
    const long long t_dx = do_dx ? static_cast<long long>(plan.dx_num_m) * plan.num_n : 0;
    const long long t_dw = do_dw ? static_cast<long long>(plan.dw_num_m) * plan.num_n : 0;
    const long long tiles = t_dx + t_dw;
    if (tiles == 0) return cudaSuccess;
    const int avail = pair ? pair_units(dev) : dev.sm_count;
    if (avail < 1) return cudaErrorInvalidConfiguration;
    const int units = static_cast<int>(tiles < avail ? tiles : avail);
    plan.sched = gemm::make_bwd_sched(static_cast<int>(t_dx), static_cast<int>(t_dw), units,
                                      plan.dx_kb, plan.dw_kb);
    if (pair) {
        if (bn == 128) return launch_width<128, true>(maps, plan, units, dev, stream);
        return launch_width<256, true>(maps, plan, units, dev, stream);
    }
    switch (bn) {
        case 128: return launch_width<128, false>(maps, plan, units, dev, stream);
        case 192: return launch_width<192, false>(maps, plan, units, dev, stream);
        default: return launch_width<256, false>(maps, plan, units, dev, stream);
    }
}

}  // namespace

int bwd_gemm_tile_n(int row_tiles_total, int cols, int sm_count, bool allow_192) {
    // Predicted time of the raster for each tile width: whole waves of
    // ceil(tiles / SMs), each as long as one tile, whose time is its width
    // divided by the MMA efficiency at that N.  Measured on B200: N = 128
    // (8 KB of shared-memory operands per 64 clocks) reaches about 0.69 of
    // the N = 256 rate; N = 192 is taken as 0.97.  Narrow tiles therefore
    // win only where they fill the last wave much better.  allow_192 = false
    // (the bf16 pair form, whose CTAs each load half the width in 64-wide
    // atoms): 256 or 128 only.
    static const int widths[3] = {256, 192, 128};
    static const double eff[3] = {1.0, 0.97, 0.69};
    int best = 256;
    double best_t = 0.0;
    for (int i = 0; i < 3; ++i) {
        if (widths[i] == 192 && !allow_192) continue;
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
    // the pair form wherever M has more than one 128-row block
    const bool pair = M > kBM && pair_units(dev) > 0;
    const int rows = pair ? 2 * kBM : kBM;
    const int bn = bwd_gemm_tile_n((M + rows - 1) / rows, K, pair ? pair_units(dev) : dev.sm_count,
                                   !pair);
    return launch_plan(dG, dU, Wg, Wu, nullptr, dX, nullptr, nullptr, M, K, N, true, false, bn,
                       pair, dev, stream);
}

cudaError_t launch_bwd_dw_bf16(const void *dG, const void *dU, const void *X, void *dWg,
                               void *dWu, int M, int K, int N, const DeviceInfo &dev,
                               cudaStream_t stream) {
    // the pair form wherever each weight matrix has more than one 128-row block
    const bool pair = N > kBM && pair_units(dev) > 0;
    const int rows = pair ? 2 * kBM : kBM;
    const int bn = bwd_gemm_tile_n(2 * ((N + rows - 1) / rows), K,
                                   pair ? pair_units(dev) : dev.sm_count, !pair);
    return launch_plan(dG, dU, nullptr, nullptr, X, nullptr, dWg, dWu, M, K, N, false, true, bn,
                       pair, dev, stream);
}

// All three in one launch: the dW tiles fill dX's tail, so the full width.
cudaError_t launch_bwd_all_bf16(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                const void *X, void *dX, void *dWg, void *dWu, int M, int K,
                                int N, const DeviceInfo &dev, cudaStream_t stream) {
    const bool pair = M > kBM && N > kBM && pair_units(dev) > 0;
    return launch_plan(dG, dU, Wg, Wu, X, dX, dWg, dWu, M, K, N, true, true, 256, pair, dev,
                       stream);
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
