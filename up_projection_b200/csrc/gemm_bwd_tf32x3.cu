// gemm_bwd_tf32x3.cu -- the backward GEMMs of the projection for fp32
// tensors, near-IEEE on the tensor cores by 3xTF32 splitting, sm_100a:
//
//   dX  [M,K] = dG Wg + dU Wu                  (reduction over N)
//   dWg [N,K] = dG^T X,   dWu [N,K] = dU^T X    (reduction over M)
//
// An fp32 training step needs these at fp32 accuracy as much as the forward
// (Liger-Kernel issue #1383, "[RFC] Testing Methodology for FP32 Convergence
// Tests on Fused SwiGLU/dSwiGLU Kernels": the fused MLP's forward and
// backward are checked together against fp32; plain TF32 fails).
//
// The operand layouts and the tile raster are those of the bf16 backward
// kernel (gemm_bwd_bf16.cu): dX accumulates both products in one accumulator
// over the 2N-long reduction [dG | dU] x [Wg ; Wu]; dW treats [dWg ; dWu] as
// one [2N x K] output.  The 3xTF32 machinery is that of the fp32 forward
// (tf32x3.cuh): each raw stage serves as hi as it landed and the split
// warps write lo beside it; per 8-deep step three kind::tf32 MMAs (lo*hi, hi*lo,
// hi*hi) accumulate into a chunk accumulator; the epilogue warps fold every
// 256-deep chunk into a running sum with round-to-nearest fp32 adds, then
// store the fp32 tile by TMA.
//
// Pair form (the output has more than one 128-row block): each MMA covers
// 256 output rows over the two CTAs of a cluster (tcgen05 cta_group::2);
// each CTA loads and splits its own 128 rows of A and half of the tile's B
// columns (16 KB per stage instead of 24 at BN = 256), its split warps
// arrive on the even CTA's ready barrier, the even CTA's warp 1 issues the
// pair's MMAs and commits each stage and chunk to the barriers of both CTAs,
// and each CTA folds and stores its own 128 rows.  The schedule below then
// runs over pairs instead of CTAs, with 256-row tiles.  (B200, LLaMA-2 13B
// M = 2048: dX alone 2.50 -> 2.19-2.28 ms, dW 2.98 -> 2.40-2.57 ms, all
// three in one launch 5.77 -> 5.03 ms; the same sums in the same order.)
//
// One launch can run dX, dW or both: a persistent grid walks a static
// schedule (gemm_common.cuh) that gives each CTA its round-robin share of the
// long dX tiles first and then fills with the short dW tiles in the order in
// which CTAs free up, so the whole backward ends in one balanced wave tail
// instead of dX's alone (at M = 2048 its 320 tiles are 2.2 waves).
//
// dX alone has no dW tiles to fill its tail, so there the tiles of the last
// partial wave (or all of them, when there are fewer tiles than SMs) are
// split along the reduction: the r tail tiles become r x S parts of
// consecutive 256-deep chunks, one per CTA after its round-robin tiles, each
// folding its chunks into its own fp32 partial tile in a workspace; a second
// kernel adds the S partials of each tile in part order (round-to-nearest
// fp32 adds, fixed order: deterministic) and writes dX.  At M = 2048,
// K = 5120 the 320 tiles become 296 whole tiles and 24 x 6 parts: 2.17
// tile-times instead of 3.
//
// fp32 operands: K-major tiles are 16 fp32 (64 bytes) per row in the 64-byte
// swizzle; MN-major tiles are atoms of 32 fp32 (128 bytes) by 16 reduction
// rows in the 128-byte swizzle with 32-byte atoms (the layout tf32 MN-major
// operands take), one TMA box {32, 16} per atom.  Output tile
// 128 x BN, MMA M=128 N=BN K=8, BN = 256, 192 or 128.  Every wait is bounded.
#include <string.h>

#include <atomic>
#include <mutex>

#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tf32x3.cuh"
#include "tmap.cuh"

namespace swiglu {

// Bit 0: a bounded wait gave up.  Read by gemm_bwd_tf32x3_status_fetch_and_clear().
__device__ unsigned int g_gemm_bwd_tf32x3_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;
using gemm::tile_coords;

constexpr int kBM = 128;                 // output rows per CTA (= MMA M per SM)
constexpr int kBR = 16;                  // reduction depth per stage
constexpr int kUmmaK = 8;                // k per tcgen05.mma, kind::tf32
constexpr int kChunkKB = 16;             // stages per accumulation chunk (256 deep)
constexpr int kSplitWarps = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * (kSplitWarps + kEpiWarps);  // 320
constexpr int kFirstSplitWarp = 2;
constexpr int kFirstEpiWarp = kFirstSplitWarp + kSplitWarps;    // 6

constexpr uint32_t kAtomBytes = 32 * kBR * 4;          // MN-major atom: 32 x 16 fp32 = 2 KB
constexpr uint32_t kABytes = kBM * kBR * 4;            // 8 KB
constexpr uint32_t kEpiBufBytes = 32 * 128;            // 32 rows x 32 fp32

// Everything that depends on the output tile width BN (= the MMA's N; 256,
// 192 or 128 columns, picked per call by the wave model of bwd_gemm_tile_n)
// and on the pair form (kPair: each MMA covers 256 output rows over the two
// CTAs of a cluster, tcgen05 cta_group::2; a CTA holds its own 128 rows of
// A and half of B's BN columns).
template <int BN, bool kPair>
struct Tile {
    static constexpr int kBN = BN;
    static constexpr int kAccCols = BN;
    static constexpr int kStages = kPair ? 6 : 4;
    static constexpr int kRows = kPair ? 2 * kBM : kBM;     // output rows per tile
    static constexpr int kBCols = kPair ? BN / 2 : BN;      // B columns this CTA loads
    // chunk accumulator + running sum, allocated as a power of two
    static constexpr int kTmemCols = 2 * BN > 256 ? 512 : 256;
    static constexpr uint32_t kBBytes = kBCols * kBR * 4;           // 16 KB at BN = 256
    static constexpr uint32_t kRawBytes = kABytes + kBBytes;        // loaded per stage
    static constexpr uint32_t kStageBytes = 2 * kRawBytes;          // + lo copies
    static constexpr uint32_t kNumBars = 3 * kStages + 3;  // full, ready, empty; chunk full/empty, drain
    static constexpr uint32_t kOffStages = 0;
    static constexpr uint32_t kOffEpi = kOffStages + kStages * kStageBytes;
    static constexpr uint32_t kOffBar = kOffEpi + kEpiWarps * kEpiBufBytes;
    static constexpr uint32_t kOffTmemPtr = kOffBar + 8 * kNumBars;
    static constexpr uint32_t kOffAbort = kOffTmemPtr + 8;
    static constexpr uint32_t kSmemBytes = kOffAbort + 8 + 1024;
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB opt-in shared memory");
    static_assert(kRawBytes % 1024 == 0, "lo copies must keep the swizzle alignment");
    static_assert(BN % 32 == 0 && kBCols % 32 == 0 && 2 * BN <= 512, "tile width");
};

// Geometry of the two tile kinds and the schedule of one launch.
struct Plan {
    int M, N, K;
    int rows;                                      // output rows per tile: 128, or 256 in pairs
    int dx_num_m, dw_row_tiles, dw_num_m, num_n;   // tiles: dx_num_m x num_n, dw_num_m x num_n
    int dx_kb, dw_kb;                              // 16-deep reduction blocks per tile
    int kb_pair;                                   // dX: blocks of one pair (dG Wg, dU Wu)
    gemm::BwdSched sched;
    // Split dX tail (dX-only launches; split.parts = 0: none): part p of
    // tail tile split.t0 + j is run by unit (CTA, or pair) j * split.parts +
    // p after its round-robin tiles and lands in workspace slot
    // j * split.parts + p (a rows x BN fp32 tile).
    gemm::DxSplit split;
};

// Tensor maps of both kinds (only those of the kinds a launch runs are used).
struct Maps {
    CUtensorMap dx_a[2];   // dG, dU: K-major {16, 128}
    CUtensorMap dx_b[2];   // Wg, Wu: MN-major atoms {32, 16}
    CUtensorMap dx_o;      // dX
    CUtensorMap dw_a[2];   // dG, dU: MN-major atoms {32, 16}
    CUtensorMap dw_b;      // X: MN-major atoms {32, 16}
    CUtensorMap dw_o[2];   // dWg, dWu
    CUtensorMap ws;        // split dX partials: [slots * rows][BN] fp32
};

struct TileInfo {
    int kind, r0, c0, num_kb, second;   // r0: this CTA's first output row
    int kb0;    // first reduction block (a split part starts inside the tile)
    int slot;   // workspace slot of a split part's partial tile, else -1
};

// The split tail (gemm_common.cuh, dx_split_shape) of a dX-only launch at
// tile width bn and `rows` output rows per tile over `units` CTAs or pairs.
inline gemm::DxSplit split_shape(int M, int K, int N, int bn, int units, int rows) {
    const long long T = static_cast<long long>((M + rows - 1) / rows) * ((K + bn - 1) / bn);
    const int kb = 2 * ((N + kBR - 1) / kBR);
    return gemm::dx_split_shape(T, (kb + kChunkKB - 1) / kChunkKB, units);
}

// The seq-th tile of unit `unit` of `units` (a CTA, or a pair of CTAs of
// which this is number `rank`).
template <int BN, bool kPair>
__device__ __forceinline__ bool next_tile(const Plan &p, int seq, TileInfo &ti, int unit,
                                          int units, int rank) {
    constexpr int kRows = Tile<BN, kPair>::kRows;
    int kind, t;
    int mt, nt;
    ti.kb0 = 0;
    ti.slot = -1;
    if (!gemm::bwd_tile_of(p.sched, unit, units, seq, kind, t)) {
        // after its round-robin tiles, a unit may take one part of a split tile
        const int slot = unit;
        int c_begin, c_end;
        if (seq != p.sched.q || !gemm::dx_split_part(p.split, slot, t, c_begin, c_end))
            return false;
        tile_coords<gemm::kGroupMBackward>(t, p.dx_num_m, p.num_n, mt, nt);
        ti.kind = gemm::kTileDx;
        ti.second = 0;
        ti.r0 = mt * kRows + rank * kBM;
        ti.c0 = nt * BN;
        ti.kb0 = c_begin * kChunkKB;
        ti.num_kb = min(p.dx_kb, c_end * kChunkKB) - ti.kb0;
        ti.slot = slot;
        return true;
    }
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
    ti.c0 = nt * BN;
    return true;
}

template <int BN, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
    swiglu_gemm_bwd_tf32x3_kernel(const __grid_constant__ Maps maps, const Plan plan) {
    using T = Tile<BN, kPair>;
    constexpr int kBN = T::kBN;
    constexpr int kAccCols = T::kAccCols;
    constexpr int kTmemCols = T::kTmemCols;
    constexpr int kStages = T::kStages;
    constexpr int kRows = T::kRows;
    constexpr int kBCols = T::kBCols;
    constexpr uint32_t kRawBytes = T::kRawBytes;
    constexpr uint32_t kStageBytes = T::kStageBytes;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);

    const uint32_t sst = base + T::kOffStages;
    const uint32_t se = base + T::kOffEpi;
    const uint32_t bar_full = base + T::kOffBar;
    const uint32_t bar_ready = bar_full + 8 * kStages;
    const uint32_t bar_empty = bar_ready + 8 * kStages;
    const uint32_t bar_cfull = bar_empty + 8 * kStages;
    const uint32_t bar_cempty = bar_cfull + 8;
    const uint32_t bar_drain = bar_cempty + 8;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(gbase + T::kOffTmemPtr);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + T::kOffAbort);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    // kPair: CTA `rank` of pair `unit`; rank 0 issues the pair's MMAs
    const int rank = kPair ? static_cast<int>(cluster_rank()) : 0;
    const int unit = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
    const int units = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_ready + 8 * s, (kPair ? 2 : 1) * kSplitWarps);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_cfull, 1);
        mbar_init(bar_cempty, (kPair ? 2 : 1) * kEpiWarps);
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
        if (plan.split.parts > 0) tma_prefetch_desc(&maps.ws);
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
        // arrive or MMA that reaches the other CTA
        cluster_sync_all();
    } else {
        __syncthreads();
    }
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_ptr);
    // kPair: the even CTA's ready / chunk-empty barriers (arrived on by both
    // CTAs), as addresses in the cluster window
    const uint32_t ready_r0 = kPair ? map_to_rank(bar_ready, 0) : 0u;
    const uint32_t cempty_r0 = kPair ? map_to_rank(bar_cempty, 0) : 0u;

    bool failed = false;
    TileInfo ti;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int seq = 0; !failed && next_tile<BN, kPair>(plan, seq, ti, unit, units, rank); ++seq) {
                for (int kb = 0; kb < ti.num_kb; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t st = sst + stage * kStageBytes;
                    mbar_arrive_expect_tx(fb, kRawBytes);
                    if (ti.kind == gemm::kTileDx) {
                        const int kba = ti.kb0 + kb;  // reduction block within the tile
                        const int pair = kba >= plan.kb_pair ? 1 : 0;
                        const int red0 = (kba - pair * plan.kb_pair) * kBR;
                        // A: [128 rows of dG or dU] x [16 of N], K-major.
                        tma_load_2d(&maps.dx_a[pair], fb, st, red0, ti.r0);
                        // B: [16 rows of Wg or Wu] x [this CTA's columns of the
                        // tile], MN-major atoms.
#pragma unroll
                        for (int j = 0; j < kBCols / 32; ++j)
                            tma_load_2d(&maps.dx_b[pair], fb, st + kABytes + j * kAtomBytes,
                                        ti.c0 + rank * kBCols + 32 * j, red0);
                    } else {
                        const int red0 = kb * kBR;
                        // A: [16 rows of M] x [128 of N] of dG or dU, MN-major.
#pragma unroll
                        for (int j = 0; j < kBM / 32; ++j)
                            tma_load_2d(&maps.dw_a[ti.second], fb, st + j * kAtomBytes,
                                        ti.r0 + 32 * j, red0);
                        // B: [16 rows of M] x [this CTA's columns] of X, MN-major.
#pragma unroll
                        for (int j = 0; j < kBCols / 32; ++j)
                            tma_load_2d(&maps.dw_b, fb, st + kABytes + j * kAtomBytes,
                                        ti.c0 + rank * kBCols + 32 * j, red0);
                    }
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
            // ------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_dx = make_idesc(2u, kRows, kBN) | kIdescBMnMajor;
            // kPair: the odd CTA's barriers, as addresses in the cluster window
            const uint32_t empty_r1 = kPair ? map_to_rank(bar_empty, 1) : 0u;
            const uint32_t cfull_r1 = kPair ? map_to_rank(bar_cfull, 1) : 0u;
            constexpr uint32_t idesc_dw = idesc_dx | kIdescAMnMajor;
            int stage = 0;
            uint32_t phase = 0;
            uint32_t chunk_phase = 0;
            for (int seq = 0; !failed && next_tile<BN, kPair>(plan, seq, ti, unit, units, rank); ++seq) {
                const bool dx = ti.kind == gemm::kTileDx;
                const uint32_t idesc = dx ? idesc_dx : idesc_dw;
                const int num_chunks = (ti.num_kb + kChunkKB - 1) / kChunkKB;
                for (int q = 0; q < num_chunks && !failed; ++q) {
                    if (!mbar_wait(bar_cempty, chunk_phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const int kb_end = min(ti.num_kb, (q + 1) * kChunkKB);
                    for (int kb = q * kChunkKB; kb < kb_end; ++kb) {
                        if (!mbar_wait(bar_ready + 8 * stage, phase, abort_flag)) {
                            failed = true;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t st = sst + stage * kStageBytes;
                        const uint64_t a_hi = dx ? sw64_kmajor_desc(st)
                                                 : sw128b32_mnmajor_desc(st, kAtomBytes);
                        const uint64_t a_lo = dx ? sw64_kmajor_desc(st + kRawBytes)
                                                 : sw128b32_mnmajor_desc(st + kRawBytes, kAtomBytes);
                        const uint64_t b_hi = sw128b32_mnmajor_desc(st + kABytes, kAtomBytes);
                        const uint64_t b_lo = sw128b32_mnmajor_desc(st + kRawBytes + kABytes, kAtomBytes);
#pragma unroll
                        for (int kk = 0; kk < kBR / kUmmaK; ++kk) {
                            // K-major: +32 B along the 64-byte swizzled row (+2);
                            // MN-major: +8 rows of 128 B (+64).
                            const uint32_t oa = dx ? 2u * kk : 64u * kk;
                            const uint32_t ob = 64u * kk;
                            const uint32_t acc = (kb == q * kChunkKB && kk == 0) ? 0u : 1u;
                            if constexpr (kPair) {
                                mma_tf32_pair(tmem_base, a_lo + oa, b_hi + ob, idesc, acc);
                                mma_tf32_pair(tmem_base, a_hi + oa, b_lo + ob, idesc, 1u);
                                mma_tf32_pair(tmem_base, a_hi + oa, b_hi + ob, idesc, 1u);
                            } else {
                                mma_tf32(tmem_base, a_lo + oa, b_hi + ob, idesc, acc);
                                mma_tf32(tmem_base, a_hi + oa, b_lo + ob, idesc, 1u);
                                mma_tf32(tmem_base, a_hi + oa, b_hi + ob, idesc, 1u);
                            }
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
                        mma_commit_pair(bar_cfull);
                        mma_commit_pair(cfull_r1);
                    } else {
                        mma_commit(bar_cfull);
                    }
                    chunk_phase ^= 1u;
                }
            }
            if constexpr (kPair)
                mma_commit_pair(bar_drain);
            else
                mma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0);
        }
    } else if (warp < kFirstEpiWarp) {
        // ---------------------------------------------------- hi/lo split
        const int sidx = threadIdx.x - 32 * kFirstSplitWarp;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        for (int seq = 0; !failed && next_tile<BN, kPair>(plan, seq, ti, unit, units, rank); ++seq) {
            for (int kb = 0; kb < ti.num_kb; ++kb) {
                if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                    failed = true;
                    break;
                }
                tf32x3::split_stage<kRawBytes, 32 * kSplitWarps>(sst + stage * kStageBytes, sidx);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (kPair)
                        mbar_arrive_remote(ready_r0 + 8 * stage);
                    else
                        mbar_arrive(bar_ready + 8 * stage);
                }
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
        for (int seq = 0; !failed && next_tile<BN, kPair>(plan, seq, ti, unit, units, rank); ++seq) {
            const int num_chunks = (ti.num_kb + kChunkKB - 1) / kChunkKB;
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
                if (lane == 0) {
                    if constexpr (kPair)
                        mbar_arrive_remote(cempty_r0);
                    else
                        mbar_arrive(bar_cempty);
                }
            }
            if (failed) break;
            const bool dx = ti.kind == gemm::kTileDx;
            const bool part = ti.slot >= 0;  // a split part: the partial tile to its slot
            const CUtensorMap *out = part ? &maps.ws : (dx ? &maps.dx_o : &maps.dw_o[ti.second]);
            const int rows = dx ? plan.M : plan.N;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
                uint32_t v[32];
                tmem_ld_32x32b_x32(run_acc + 32u * c, v);
                tmem_ld_wait(v);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    sts_v4(buf + static_cast<uint32_t>(lane) * 128u +
                               ((static_cast<uint32_t>(j) ^ swz) << 4),
                           make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int x = part ? c * 32 : ti.c0 + c * 32;
                    const int y = part ? ti.slot * kRows + rank * kBM + quad * 32
                                       : ti.r0 + quad * 32;
                    if (part || (x < plan.K && y < rows)) {
                        tma_store_2d(out, buf, x, y);
                        bulk_commit();
                    }
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
    }

    if (failed) atomicOr(&g_gemm_bwd_tf32x3_status, 1u);

    tc_fence_before();
    __syncthreads();
    // kPair: the pair's MMAs have completed (the issuer drained them) and
    // both CTAs' epilogues are done before either frees TMEM or leaves
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

// dX of the split tail tiles: for every element the parts' partial sums are
// added in part order with round-to-nearest fp32 adds (a fixed order, so the
// result does not depend on which CTA finished first), then stored if inside
// dX.  Four consecutive columns per thread.
__global__ void __launch_bounds__(256)
    bwd_dx_split_combine_kernel(const float *__restrict__ ws, float *__restrict__ dX,
                                const Plan plan, int bn) {
    const int q4 = bn / 4;                           // float4 per partial row
    const int rows = plan.rows;                      // partial rows per tile
    const long long per_tile = static_cast<long long>(rows) * q4;
    const long long total = per_tile * plan.split.tiles;
    const int S = plan.split.parts;
    for (long long idx = blockIdx.x * 256ll + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * 256) {
        const int j = static_cast<int>(idx / per_tile);
        const int rem = static_cast<int>(idx - j * per_tile);
        const int i = rem / q4, c = (rem - i * q4) * 4;
        int mt, nt;
        tile_coords<gemm::kGroupMBackward>(plan.split.t0 + j, plan.dx_num_m, plan.num_n, mt, nt);
        const int row = mt * rows + i, col = nt * bn + c;
        if (row >= plan.M || col >= plan.K) continue;
        const float4 *p = reinterpret_cast<const float4 *>(ws) +
                          (static_cast<long long>(j) * S * rows + i) * q4 + c / 4;
        float4 acc = p[0];
        for (int s = 1; s < S; ++s) {
            const float4 v = p[static_cast<long long>(s) * rows * q4];
            acc.x = __fadd_rn(acc.x, v.x);
            acc.y = __fadd_rn(acc.y, v.y);
            acc.z = __fadd_rn(acc.z, v.z);
            acc.w = __fadd_rn(acc.w, v.w);
        }
        float *o = dX + static_cast<long long>(row) * plan.K + col;
        const float a[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (col + e < plan.K) o[e] = a[e];
    }
}

std::atomic<unsigned> g_attr_set_mask[6];

template <int BN, bool kPair>
cudaError_t set_smem_attr(const DeviceInfo &dev) {
    constexpr int idx = (BN == 256 ? 0 : (BN == 192 ? 1 : 2)) + (kPair ? 3 : 0);
    const unsigned bit = 1u << (dev.device & 31);
    if (!(g_attr_set_mask[idx].load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(swiglu_gemm_bwd_tf32x3_kernel<BN, kPair>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(Tile<BN, kPair>::kSmemBytes));
        if (e != cudaSuccess) return e;
        g_attr_set_mask[idx].fetch_or(bit);
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
template <int BN, bool kPair>
cudaError_t launch_bn(const Maps &maps, const Plan &plan, int units, const DeviceInfo &dev,
                      cudaStream_t stream) {
    cudaError_t e = set_smem_attr<BN, kPair>(dev);
    if (e != cudaSuccess) return e;
    if constexpr (kPair) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(2 * units));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = Tile<BN, kPair>::kSmemBytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        set_cluster_attr(attr[0]);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, swiglu_gemm_bwd_tf32x3_kernel<BN, kPair>, maps, plan);
        if (e != cudaSuccess) return e;
    } else {
        swiglu_gemm_bwd_tf32x3_kernel<BN, kPair>
            <<<units, kThreads, Tile<BN, kPair>::kSmemBytes, stream>>>(maps, plan);
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
        cfg.dynamicSmemBytes = Tile<256, true>::kSmemBytes;
        cudaLaunchAttribute attr[1];
        set_cluster_attr(attr[0]);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, swiglu_gemm_bwd_tf32x3_kernel<256, true>, &cfg) ==
                cudaSuccess && n > 0)
            u = n;
        else
            (void)cudaGetLastError();
    }
    g_pair_units[dev.device].store(u);
    return u > 0 ? u : 0;
}

// Encodes the maps of the kinds requested (null pointers: kind not run) and
// launches one persistent grid over all their tiles, `bn` columns wide.
// pair: the pair form (256-row tiles, a pair of SMs per tile).
// split_parts > 0 (dX only; it must be the parts of split_shape at this
// width and form): the tail tiles' partials go to `ws` (tiles x parts x
// rows x bn fp32), which the combine kernel then reduces into dX.
cudaError_t launch_plan(const void *dG, const void *dU, const void *Wg, const void *Wu,
                        const void *X, void *dX, void *dWg, void *dWu, int M, int K, int N,
                        bool do_dx, bool do_dw, int bn, bool pair, int split_parts, void *ws,
                        const DeviceInfo &dev, cudaStream_t stream) {
    if (bn != 256 && bn != 192 && bn != 128) return cudaErrorInvalidValue;
    const int units = pair ? pair_units(dev) : dev.sm_count;
    if (units < 1) return cudaErrorInvalidConfiguration;
    const int rows = pair ? 2 * kBM : kBM;
    const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const CUtensorMapSwizzle sw64 = CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapSwizzle sw128 = CU_TENSOR_MAP_SWIZZLE_128B;
    const CUtensorMapSwizzle mn = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;
    const uint64_t n_bytes = static_cast<uint64_t>(N) * 4, k_bytes = static_cast<uint64_t>(K) * 4;
    Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (do_dx &&
        (!encode_tmap_2d(&maps.dx_a[0], dG, f32, N, M, n_bytes, kBR, kBM, sw64) ||
         !encode_tmap_2d(&maps.dx_a[1], dU, f32, N, M, n_bytes, kBR, kBM, sw64) ||
         !encode_tmap_2d(&maps.dx_b[0], Wg, f32, K, N, k_bytes, 32, kBR, mn) ||
         !encode_tmap_2d(&maps.dx_b[1], Wu, f32, K, N, k_bytes, 32, kBR, mn) ||
         !encode_tmap_2d(&maps.dx_o, dX, f32, K, M, k_bytes, 32, 32, sw128)))
        return cudaErrorInvalidValue;
    if (do_dw &&
        (!encode_tmap_2d(&maps.dw_a[0], dG, f32, N, M, n_bytes, 32, kBR, mn) ||
         !encode_tmap_2d(&maps.dw_a[1], dU, f32, N, M, n_bytes, 32, kBR, mn) ||
         !encode_tmap_2d(&maps.dw_b, X, f32, K, M, k_bytes, 32, kBR, mn) ||
         !encode_tmap_2d(&maps.dw_o[0], dWg, f32, K, N, k_bytes, 32, 32, sw128) ||
         !encode_tmap_2d(&maps.dw_o[1], dWu, f32, K, N, k_bytes, 32, 32, sw128)))
        return cudaErrorInvalidValue;
    Plan plan{};
    plan.M = M;
    plan.N = N;
    plan.K = K;
    plan.rows = rows;
    plan.num_n = (K + bn - 1) / bn;
    plan.dx_num_m = (M + rows - 1) / rows;
    plan.dw_row_tiles = (N + rows - 1) / rows;
    plan.dw_num_m = 2 * plan.dw_row_tiles;
    plan.kb_pair = (N + kBR - 1) / kBR;
    plan.dx_kb = 2 * plan.kb_pair;
    plan.dw_kb = (M + kBR - 1) / kBR;
    long long t_dx = do_dx ? static_cast<long long>(plan.dx_num_m) * plan.num_n : 0;
    const long long t_dw = do_dw ? static_cast<long long>(plan.dw_num_m) * plan.num_n : 0;
    const long long tiles = t_dx + t_dw;
    if (tiles == 0) return cudaSuccess;
    int grid = static_cast<int>(tiles < units ? tiles : units);   // units launched
    if (split_parts > 0) {
        if (do_dw || ws == nullptr) return cudaErrorInvalidValue;
        const gemm::DxSplit sp = split_shape(M, K, N, bn, units, rows);
        if (sp.parts != split_parts) return cudaErrorInvalidValue;
        plan.split = sp;
        t_dx = sp.t0;  // the round-robin tiles: whole waves
        grid = units;
        if (!encode_tmap_2d(&maps.ws, ws, f32, static_cast<uint64_t>(bn),
                            static_cast<uint64_t>(sp.tiles) * sp.parts * rows,
                            static_cast<uint64_t>(bn) * 4, 32, 32, sw128))
            return cudaErrorInvalidValue;
    }
    plan.sched = gemm::make_bwd_sched(static_cast<int>(t_dx), static_cast<int>(t_dw), grid,
                                      plan.dx_kb, plan.dw_kb);
    cudaError_t e;
    if (pair) {
        if (bn == 256) e = launch_bn<256, true>(maps, plan, grid, dev, stream);
        else if (bn == 192) e = launch_bn<192, true>(maps, plan, grid, dev, stream);
        else e = launch_bn<128, true>(maps, plan, grid, dev, stream);
    } else {
        if (bn == 256) e = launch_bn<256, false>(maps, plan, grid, dev, stream);
        else if (bn == 192) e = launch_bn<192, false>(maps, plan, grid, dev, stream);
        else e = launch_bn<128, false>(maps, plan, grid, dev, stream);
    }
    if (e != cudaSuccess || split_parts == 0) return e;
    const long long vec = static_cast<long long>(plan.split.tiles) * rows * (bn / 4);
    const long long blocks = (vec + 255) / 256;
    const int cgrid = static_cast<int>(blocks < 4ll * dev.sm_count ? blocks : 4ll * dev.sm_count);
    bwd_dx_split_combine_kernel<<<cgrid, 256, 0, stream>>>(static_cast<const float *>(ws),
                                                         static_cast<float *>(dX), plan, bn);
    return cudaGetLastError();
}

}  // namespace

DxSplitPlan dx_split_plan(int M, int K, int N, const DeviceInfo &dev) {
    // Predicted time of each (width, split): whole rounds of tiles, each
    // tile its chunk count times one chunk's time at that width (B200, 13B
    // shape: ~12 us per 256-deep chunk of a 128 x 256 tile; 192-wide tiles
    // run at 0.83 of that rate per column, 128-wide taken as 0.6), and with a
    // split one part's chunks plus the combine kernel (a launch and a pass
    // over the partials).
    static const int widths[3] = {256, 192, 128};
    static const double eff[3] = {1.0, 0.83, 0.6};
    constexpr double kChunkUs = 12.0;
    // The pair form wherever M has more than one 128-row block: 256-row
    // tiles over the pairs that can be resident at once.
    const bool pair = M > kBM && pair_units(dev) > 0;
    const int sm_count = pair ? pair_units(dev) : dev.sm_count;   // units
    const int tile_rows = pair ? 2 * kBM : kBM;
    DxSplitPlan best{256, 0, 0, pair};
    double best_t = -1.0;
    const long long rows = (M + tile_rows - 1) / tile_rows;
    if (rows <= 0 || K <= 0 || sm_count < 1) return best;
    for (int i = 0; i < 3; ++i) {
        const int w = widths[i];
        const long long T = rows * ((K + w - 1) / w);
        const gemm::DxSplit sp = split_shape(M, K, N, w, sm_count, tile_rows);
        const double chunk = kChunkUs * w / 256.0 / eff[i];
        const double tile = sp.chunks * chunk;
        const double t_plain = static_cast<double>((T + sm_count - 1) / sm_count) * tile;
        if (best_t < 0.0 || t_plain < best_t) {
            best = DxSplitPlan{w, 0, 0, pair};
            best_t = t_plain;
        }
        if (sp.parts > 0) {
            const size_t bytes = static_cast<size_t>(sp.tiles) * sp.parts * tile_rows * w * 4;
            const double t_split = static_cast<double>(T / sm_count) * tile +
                                   ((sp.chunks + sp.parts - 1) / sp.parts) * chunk + 4.0 +
                                   static_cast<double>(bytes) / 3.0e6;
            if (t_split < best_t) {
                best = DxSplitPlan{w, sp.parts, bytes, pair};
                best_t = t_split;
            }
        }
    }
    return best;
}

namespace {
std::mutex g_ws_pool_mu;
cudaMemPool_t g_ws_pool[64];

// The memory pool the split workspaces come from: one per device, created by
// the library, that keeps the memory it has mapped between calls.  (The
// device's default pool returns its memory at every synchronisation, and a
// call after one then maps its workspace again: up to a few hundred us.)
cudaError_t workspace_pool(int device, cudaMemPool_t *out) {
    if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_ws_pool_mu);
    if (g_ws_pool[device] == nullptr) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = device;
        cudaMemPool_t pool = nullptr;
        cudaError_t e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            (void)cudaMemPoolDestroy(pool);
            return e;
        }
        g_ws_pool[device] = pool;
    }
    *out = g_ws_pool[device];
    return cudaSuccess;
}
}  // namespace

// dX alone: the tile width and split of the cost model (dx_split_plan);
// with a split, a workspace for the partial tiles is taken from the
// library's pool for the device on `stream` and released after the combine
// kernel, both in stream order.
cudaError_t launch_bwd_dx_tf32x3(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                 void *dX, int M, int K, int N, const DeviceInfo &dev,
                                 cudaStream_t stream) {
    const DxSplitPlan sp = dx_split_plan(M, K, N, dev);
    if (sp.parts == 0)
        return launch_plan(dG, dU, Wg, Wu, nullptr, dX, nullptr, nullptr, M, K, N, true, false,
                           sp.bn, sp.pair, 0, nullptr, dev, stream);
    cudaMemPool_t pool = nullptr;
    cudaError_t e = workspace_pool(dev.device, &pool);
    if (e != cudaSuccess) return e;
    void *ws = nullptr;
    e = cudaMallocFromPoolAsync(&ws, sp.workspace_bytes, pool, stream);
    if (e != cudaSuccess) return e;
    e = launch_plan(dG, dU, Wg, Wu, nullptr, dX, nullptr, nullptr, M, K, N, true, false, sp.bn,
                    sp.pair, sp.parts, ws, dev, stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : f;
}

// ---------------------------------------------------------------------------
// dX alone without any allocation, for swiglu_bwd_dx_noalloc: the split
// tail's partial tiles go to a fixed array in device memory instead of a
// workspace from the memory pool.  The split never needs more than one
// partial tile per unit -- 128 x 256 fp32 per CTA, or 256 x 256 per pair of
// CTAs -- so the bytes of 148 single-CTA tiles (an SM each on B200) cover
// every shape there; a plan that would need more (a GPU with more SMs) is
// refused.  Nothing in it must start at zero: each slot a call
// reads was written earlier in the same call.  Every GPU that loads this
// library holds the array until the process exits, and all calls on a GPU
// share it.
constexpr size_t kStaticScratchBytes = 148ull * kBM * 256 * 4;  // 18.5 MiB
static __device__ __align__(256) unsigned char g_dx_static_scratch[kStaticScratchBytes];

namespace {
// The array's device address, looked up once per device (host code only
// knows a host-side stand-in for the symbol).
std::atomic<void *> g_dx_static_scratch_ptr[64];
}  // namespace

cudaError_t launch_bwd_dx_tf32x3_static(const void *dG, const void *dU, const void *Wg,
                                        const void *Wu, void *dX, int M, int K, int N,
                                        const DeviceInfo &dev, cudaStream_t stream,
                                        bool *scratch_too_small) {
    *scratch_too_small = false;
    const DxSplitPlan sp = dx_split_plan(M, K, N, dev);
    if (sp.parts == 0)
        return launch_plan(dG, dU, Wg, Wu, nullptr, dX, nullptr, nullptr, M, K, N, true, false,
                           sp.bn, sp.pair, 0, nullptr, dev, stream);
    if (sp.workspace_bytes > kStaticScratchBytes) {
        *scratch_too_small = true;
        return cudaErrorInvalidValue;
    }
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    void *ws = g_dx_static_scratch_ptr[dev.device].load();
    if (ws == nullptr) {
        // set-up on this device's first call (the device is current here)
        const cudaError_t e = cudaGetSymbolAddress(&ws, g_dx_static_scratch);
        if (e != cudaSuccess) return e;
        g_dx_static_scratch_ptr[dev.device].store(ws);
    }
    return launch_plan(dG, dU, Wg, Wu, nullptr, dX, nullptr, nullptr, M, K, N, true, false, sp.bn,
                       sp.pair, sp.parts, ws, dev, stream);
}

cudaError_t launch_bwd_dw_tf32x3(const void *dG, const void *dU, const void *X, void *dWg,
                                 void *dWu, int M, int K, int N, const DeviceInfo &dev,
                                 cudaStream_t stream) {
    // the pair form wherever each weight matrix has more than one 128-row block
    const bool pair = N > kBM && pair_units(dev) > 0;
    const int rows = pair ? 2 * kBM : kBM;
    const int bn = bwd_gemm_tile_n(2 * ((N + rows - 1) / rows), K,
                                   pair ? pair_units(dev) : dev.sm_count);
    return launch_plan(dG, dU, nullptr, nullptr, X, nullptr, dWg, dWu, M, K, N, false, true, bn,
                       pair, 0, nullptr, dev, stream);
}

// All three in one launch: the dW tiles fill dX's tail, so the full width.
cudaError_t launch_bwd_all_tf32x3(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                  const void *X, void *dX, void *dWg, void *dWu, int M, int K,
                                  int N, const DeviceInfo &dev, cudaStream_t stream) {
    const bool pair = M > kBM && N > kBM && pair_units(dev) > 0;
    return launch_plan(dG, dU, Wg, Wu, X, dX, dWg, dWu, M, K, N, true, true, 256, pair, 0, nullptr,
                       dev, stream);
}

cudaError_t gemm_bwd_tf32x3_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_gemm_bwd_tf32x3_status,
                                              sizeof(unsigned int), 0, cudaMemcpyDeviceToHost,
                                              stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gemm_bwd_tf32x3_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
