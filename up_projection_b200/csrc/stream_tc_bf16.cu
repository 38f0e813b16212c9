// stream_tc_bf16.cu -- fused SwiGLU forward for batched-decode M (9..128),
// bf16, as a weight stream through the tcgen05 tensor cores.
//
// With a few dozen rows of X the op is still a read of Wg and Wu from HBM
// once (AstrAI swiglu_benchmark.md, "HBM re-measurement and kernel
// simplification": the fused kernel's target is the cold-read floor of both
// weight matrices), but the dot products outgrow warp-level mma.sync.  Here
// they run on tcgen05 with the operands swapped against the dual GEMM:
//
//  * A (the MMA's M = 64 or 128 rows) is a k-slice of X; rows >= M are
//    zero-filled by the copy or lie beyond the X box (their TMEM lanes are
//    never read);
//  * B (the MMA's N) is the CTA's own rows of Wg, and in a second MMA the
//    same rows of Wu.  D_g lane m, column c = g(m, n0 + c) and D_u the same
//    for u, so the activation and gate product are lane-local.
//
// A CTA owns a contiguous, balanced range of cnt units of 8 output columns
// (within one unit of even over the SMs): rows 8 u0 .. 8 (u0 + cnt) of each
// weight matrix are consecutive.  Per k-slice ONE TMA box covers them in both
// matrices: a 4-D view [k/64][matrix][rows][64] whose matrix stride is the
// distance between the two weight buffers lands as [k-block][Wg rows; Wu rows]
// [128 B] -- per k-block one run of 1024-byte 128-byte-swizzle atoms, the
// K-major operand layout -- so ONE MMA per k16 step computes gate and up
// together (N = 16 cnt).  (Where that view does not exist -- Wg == Wu, or
// buffers 1 TB apart -- two 3-D boxes and two MMAs per step do the same.)
// The X box of the slice rides in the same ring stage.  Per-CTA unit counts
// differ by at most one, so two tensor maps (box heights 8 q and 8 (q + 1))
// serve every CTA.
// The k16 steps alternate between two accumulator sets, each issued by its
// own thread (no MMA waits on its predecessor's accumulator, and two threads
// keep the tensor pipe fed); the epilogue sums them, forms
// h = act(alpha g) u in fp32 and rounds once to bf16 -- spread over all 192
// threads through shared memory when few warps hold the rows.
// Where a CTA's stages are small enough two CTAs share an SM, so that one's
// tail overlaps the other's stream (and, with weights_stable, the next
// call's weight prefetch).
//
// Waits are bounded; a stuck pipeline sets the status word, the MMAs and
// copies in flight are drained and TMEM is freed before the kernel returns.
#include <cuda_bf16.h>

#include <atomic>

#include "activation.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace swiglu {

// Status word of this translation unit's kernel (bit 0 = a wait gave up).
__device__ unsigned int g_stream_tc_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;

constexpr int kThreads = 192;   // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 epilogue
constexpr int kMaxRing = 8;
constexpr int kMaxSmem = 227 * 1024;
constexpr int kNumBars = 2 * kMaxRing + 3;  // full, empty, acc, drain[2]
// barriers, then abort flag (+0), TMEM slot (+16), epilogue flag (+32); alignment
constexpr int kTail = 8 * kNumBars + 64 + 1024;

struct StreamGeo {
    int mpad;      // X rows per box (M rounded up to 8)
    int mma_m;     // 64 when mpad <= 64, else 128
    int q1;        // most units per CTA (box height 8 q1)
    int region;    // TMEM columns of one accumulator region (8 q1, rounded to 16)
    int kb;        // 64-wide k-blocks per slice
    int kblocks;   // K / 64
    int slices;    // ceil(kblocks / kb)
    int ring;      // stages
    int wbytes;    // space of one weight box in a stage: q1 * kb * 1024
    int stage;     // 2 wbytes + mpad * kb * 128
    int off_bar, smem;
    int tmem_cols;
    int epi_units;  // units per epilogue chunk: mpad x 64 B each fit the ring
    int ctas_per_sm;
    bool ok;
};

// Stage layout for units_per_cta = q1 within `budget` bytes: the largest
// slice (16 .. 1 k-blocks, at most K) with a ring of >= min_ring stages.
// Behind the ring: slack for the A operand's rows beyond the X box, then
// the barriers.
inline StreamGeo stream_geometry(int M, int K, int q1, int budget, int min_ring) {
    StreamGeo g{};
    g.ok = false;
    if (M < 1 || K < 64 || K % 64 != 0 || q1 < 1 || q1 > 32) return g;
    g.mpad = (M + 7) / 8 * 8;
    if (g.mpad > 128) return g;
    g.mma_m = g.mpad <= 64 ? 64 : 128;
    g.q1 = q1;
    g.region = (8 * q1 + 15) / 16 * 16;
    g.kblocks = K / 64;
    const int slack = (g.mma_m - g.mpad) * 128;
    static const int kCandidates[] = {16, 12, 8, 6, 4, 3, 2, 1};
    for (int kb : kCandidates) {
        if (kb > g.kblocks) kb = g.kblocks;  // no slice longer than K
        const int stage = kb * 128 * (16 * q1 + g.mpad);
        const int room = budget - slack - kTail;
        if (room < min_ring * stage) continue;
        g.kb = kb;
        g.stage = stage;
        g.wbytes = q1 * kb * 1024;
        g.ring = room / stage > kMaxRing ? kMaxRing : room / stage;
        g.ok = true;
        break;
    }
    if (!g.ok) return g;
    g.slices = (g.kblocks + g.kb - 1) / g.kb;
    g.off_bar = g.ring * g.stage + slack;
    g.smem = g.off_bar + kTail;
    int cols = 32;
    while (cols < 4 * g.region) cols *= 2;
    g.tmem_cols = cols;
    g.epi_units = (g.ring * g.stage) / (g.mpad * 64);
    if (g.epi_units > q1) g.epi_units = q1;
    if (g.epi_units < 1) g.ok = false;
    if (g.smem > kMaxSmem || cols > 512) g.ok = false;
    return g;
}

struct StreamPlan {
    StreamGeo geo;
    int grid;
    int q;          // units of the smaller CTAs (q1 = q or q + 1)
};

// Two CTAs per SM (half the shared memory and TMEM each) when the stages
// still hold weight boxes of >= 4 KB in a ring of >= 3; else one CTA per SM
// (more CTAs, in waves, where an SM's share would exceed 16 units).  (Swept
// on B200: 8 KB instead of 4 KB costs 16 % at AstrAI-1B M = 64; no threshold
// costs 4 % at M = 128; a ring of >= 4 costs up to 20 %.)
inline StreamPlan stream_plan(int M, int K, int N, int sm_count) {
    StreamPlan p{};
    p.geo.ok = false;
    const int units = N / 8;
    if (units < 1 || sm_count < 1) return p;
    for (int cps = 2; cps >= 1; --cps) {
        const int max_units = 16 / cps;
        int grid = units < sm_count * cps ? units : sm_count * cps;
        const int need = (units + max_units - 1) / max_units;
        if (grid < need) {
            if (cps == 2) continue;
            grid = need;
        }
        const int q1 = (units + grid - 1) / grid;
        const int budget = cps == 2 ? 110 * 1024 : 220 * 1024;
        StreamGeo g = stream_geometry(M, K, q1, budget, 3);
        if (cps == 2 && (!g.ok || g.wbytes < 4 * 1024)) continue;
        if (!g.ok) g = stream_geometry(M, K, q1, budget, 2);
        if (!g.ok) return p;
        g.ctas_per_sm = cps;
        p.geo = g;
        p.grid = grid;
        p.q = units / grid;
        return p;
    }
    return p;
}

__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Barrier `id` (1..15) over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// tm_w*_lo: box height 8 q (CTAs with q units), tm_w*_hi: 8 (q + 1).  pair:
// tm_wg_* are the 4-D views over both matrices (matrix 0 the lower address;
// swapped: that is Wu) and tm_wu_* are unused.
__global__ void __launch_bounds__(kThreads, 1)
    swiglu_stream_tc_bf16_kernel(const __grid_constant__ CUtensorMap tm_x,
                                 const __grid_constant__ CUtensorMap tm_wg_lo,
                                 const __grid_constant__ CUtensorMap tm_wu_lo,
                                 const __grid_constant__ CUtensorMap tm_wg_hi,
                                 const __grid_constant__ CUtensorMap tm_wu_hi, int q,
                                 int pair, int swapped,
                                 __nv_bfloat16 *__restrict__ H, int M, int N, int weights_stable,
                                 int which_act, float alpha, __nv_bfloat16 *__restrict__ Gout,
                                 __nv_bfloat16 *__restrict__ Uout, const StreamGeo geo,
                                 const void *__restrict__ X, uint32_t x_bytes) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int units = N / 8;
    const int u_begin = static_cast<int>((static_cast<long long>(units) * blockIdx.x) / gridDim.x);
    const int u_end = static_cast<int>((static_cast<long long>(units) * (blockIdx.x + 1)) / gridDim.x);
    const int cnt = u_end - u_begin;  // q or q + 1
    const CUtensorMap *tm_wg = cnt > q ? &tm_wg_hi : &tm_wg_lo;
    const CUtensorMap *tm_wu = cnt > q ? &tm_wu_hi : &tm_wu_lo;
    if (threadIdx.x == 0) {
        tma_prefetch_desc(tm_wg);
        if (!pair) tma_prefetch_desc(tm_wu);
        tma_prefetch_desc(&tm_x);
        // X is read only after the dependency wait; the first CTA to start
        // brings it into L2 now (it may have been evicted by the weights
        // streamed since its last use).
        if (weights_stable && blockIdx.x == 0) bulk_prefetch_l2(X, x_bytes);
    }
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (sbase - raw);
    const uint32_t bar_full = sbase + geo.off_bar;
    const uint32_t bar_empty = bar_full + 8 * kMaxRing;
    const uint32_t bar_acc = bar_empty + 8 * kMaxRing;
    const uint32_t bar_drain = bar_acc + 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + geo.off_bar + 8 * kNumBars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + geo.off_bar + 8 * kNumBars + 16);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < geo.ring; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 2);  // one commit per MMA issuer
        }
        mbar_init(bar_acc, 2);
        mbar_init(bar_drain, 1);
        mbar_init(bar_drain + 8, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(geo.tmem_cols));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    // Programmatic dependent launch: the next call may start prefetching its
    // weights while this one finishes (it waits for this grid before X).
    // Triggered only once this CTA holds its TMEM columns, so that a next
    // call's CTA on the same SM can never take them first and leave this
    // CTA's allocation waiting on a grid that in turn waits for this one.
    if (weights_stable) griddep_launch_dependents();

    bool failed = false;
    // ----------------------------------------------------- MMA issuers
    // D (TMEM columns): accumulator set p at [2pR, 2pR + 2R); set p takes the
    // k16 steps kk = p, p + 2 of every k-block and is issued by its own
    // thread (warp 1 lane 0: set 0; warp 2 lane 0: set 1), so that two
    // threads keep the tensor pipe fed.  pair: one MMA writes [matrix 0 |
    // matrix 1] (N = 16 cnt).  Split: gate at [0, R), up at [R, 2R) of the
    // set; for M = 128 the MMA's N is a multiple of 16, so an odd cnt reads 8
    // rows past its box (columns never read).  Each issuer commits to the
    // stage's empty barrier (two arrivals free it) and to the accumulator
    // barrier (two arrivals), and drains its own MMAs before TMEM is freed.
    auto run_mma = [&](int p) {
        const int n_mma = pair ? 16 * cnt
                               : (geo.mma_m == 128 ? (8 * cnt + 15) / 16 * 16 : 8 * cnt);
        const uint32_t idesc = make_idesc(1u, static_cast<uint32_t>(geo.mma_m),
                                          static_cast<uint32_t>(n_mma));
        const uint32_t R = static_cast<uint32_t>(geo.region);
        const uint32_t d = tmem_base + static_cast<uint32_t>(p) * 2u * R;
        const uint32_t drain = bar_drain + 8 * p;
        int stage = 0;
        uint32_t phase = 0;
        for (int j = 0; j < geo.slices && !failed; ++j) {
            if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const uint32_t st = sbase + stage * geo.stage;
            const uint32_t xs = st + 2 * geo.wbytes;
            const int left = geo.kblocks - j * geo.kb;
            const int nbv = left < geo.kb ? left : geo.kb;
            for (int b = 0; b < nbv; ++b) {
                const uint64_t ad = sw128_kmajor_desc(xs + b * geo.mpad * 128);
                const uint32_t acc = (j > 0 || b > 0) ? 1u : 0u;
                if (pair) {
                    // block b: [matrix 0 rows; matrix 1 rows], 2 cnt atoms
                    const uint64_t bw = sw128_kmajor_desc(st + b * cnt * 2048);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // +32 bytes along k inside the swizzled row per k16
                        const uint32_t kk = static_cast<uint32_t>(p + 2 * h);
                        mma_f16(d, ad + 2u * kk, bw + 2u * kk, idesc, h == 0 ? acc : 1u);
                    }
                } else {
                    const uint64_t bg = sw128_kmajor_desc(st + b * cnt * 1024);
                    const uint64_t bu = sw128_kmajor_desc(st + geo.wbytes + b * cnt * 1024);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t kk = static_cast<uint32_t>(p + 2 * h);
                        const uint32_t a = h == 0 ? acc : 1u;
                        mma_f16(d, ad + 2u * kk, bg + 2u * kk, idesc, a);
                        mma_f16(d + R, ad + 2u * kk, bu + 2u * kk, idesc, a);
                    }
                }
            }
            mma_commit(bar_empty + 8 * stage);
            if (++stage == geo.ring) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (failed) *abort_flag = 1;
        else mma_commit(bar_acc);
        // Every MMA issued here must finish before TMEM is released.
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
    };
    if (warp == 0) {
        if (lane == 0 && cnt > 0) {
            // ------------------------------------------------ TMA producer
            // stage: [weights: pair box [kb][2][8 cnt][64], or Wg box then
            //         Wu box (wbytes apart)][X box [kb][mpad][64]]
            const uint32_t tx = static_cast<uint32_t>(geo.kb * 128 * (16 * cnt + geo.mpad));
            const int row = 8 * u_begin;
            auto issue_x = [&](int j) {
                const int s = j % geo.ring;
                const uint32_t st = sbase + s * geo.stage;
                // rows >= M and k-blocks beyond K are zero-filled
                tma_load_3d(&tm_x, bar_full + 8 * s, st + 2 * geo.wbytes, 0, 0, j * geo.kb);
            };
            // With weights_stable the first stages' weights are requested
            // before waiting for the work that produces X.
            const int deferred = weights_stable ? (geo.ring < geo.slices ? geo.ring : geo.slices) : 0;
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int j = 0; j < geo.slices; ++j) {
                if (j == deferred && deferred > 0) {
                    griddep_wait();
                    for (int jj = 0; jj < deferred; ++jj) issue_x(jj);
                }
                if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                    failed = true;
                    break;
                }
                const uint32_t fb = bar_full + 8 * stage;
                const uint32_t st = sbase + stage * geo.stage;
                mbar_arrive_expect_tx(fb, tx);
                if (pair) {
                    tma_load_4d(tm_wg, fb, st, 0, row, 0, j * geo.kb);
                } else {
                    tma_load_3d(tm_wg, fb, st, 0, row, j * geo.kb);
                    tma_load_3d(tm_wu, fb, st + geo.wbytes, 0, row, j * geo.kb);
                }
                if (j >= deferred) issue_x(j);
                ++issued;
                if (++stage == geo.ring) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!failed && deferred > 0 && deferred == geo.slices) {
                griddep_wait();
                for (int jj = 0; jj < deferred; ++jj) issue_x(jj);
            }
            if (failed) *abort_flag = 1;
            // Never leave while a copy issued here may still write shared
            // memory.  (A failure can only occur after the deferred X copies
            // were issued: the first `deferred` stages wait on nothing.)
            for (int s = 0; s < geo.ring; ++s) {
                if (issued > s) {
                    const int uses = (issued - 1 - s) / geo.ring + 1;
                    mbar_wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && cnt > 0) run_mma(0);
    }
    __syncwarp();  // warps 0 and 1 reconverge and join the epilogue
    {
        // ------------------------------------------------------- epilogue
        // M = 128 MMA (M > 64): every quadrant's warp holds 32 rows and
        // forms h for them directly from TMEM, 16-byte stores per unit.
        // M = 64 MMA: the warps holding D rows (16 per quadrant, a single
        // warp at M <= 16) copy g and u (both accumulator sets summed) from
        // TMEM to shared memory -- the ring, idle once every MMA has
        // completed -- and then all 192 threads (the copy and MMA warps
        // join once their roles end) form the activations and store H, two
        // columns each, so that serial activations in few lanes do not
        // become the kernel's tail (B200, AstrAI-1B M = 16: 11.7 -> 10.2 us
        // with the 128 epilogue threads, M = 64: 10.96 -> 10.76 us with all
        // 192; at M = 128 the round trip costs more than it saves).  Units
        // go through in chunks that fit the ring.  Only warps 2..5 touch
        // TMEM (warp w may read lanes 32 (w mod 4) .. +31).
        const int et = threadIdx.x;  // 0..191
        const int quad = warp & 3;        // TMEM lane quadrant this warp may read
        // D row m sits in lane m (M = 128 MMA), or for M = 64 in lanes 0..15
        // of each quadrant: row 16 quad + lane.
        const int rows_per_quad = geo.mma_m == 64 ? 16 : 32;
        const int m_lane = lane < rows_per_quad ? quad * rows_per_quad + lane : M;
        volatile int *epi_ok =
            reinterpret_cast<volatile int *>(gbase + geo.off_bar + 8 * kNumBars + 32);
        if (warp == 2 && lane == 0 && cnt > 0) run_mma(1);
        if (warp == 2 && lane == 0) {
            const bool ok = cnt > 0 && !failed && mbar_wait(bar_acc, 0, abort_flag);
            if (cnt > 0 && !ok) failed = true;
            *epi_ok = ok ? 1 : 0;
        }
        named_bar_sync(1, kThreads);
        if (*epi_ok) {
            tc_fence_after();
            const uint32_t R = static_cast<uint32_t>(geo.region);
            const uint32_t row_off = static_cast<uint32_t>(quad * 32) << 16;
            // column offsets of gate and up within an accumulator set
            const uint32_t c8 = static_cast<uint32_t>(8 * cnt);
            const uint32_t goff = pair ? (swapped ? c8 : 0u) : 0u;
            const uint32_t uoff = pair ? (swapped ? 0u : c8) : R;
            float *E = reinterpret_cast<float *>(gbase);  // [m][unit][g 8, u 8]
            if (geo.mma_m == 128) {
                for (int i = 0; i < cnt && warp >= 2 && quad * rows_per_quad < M; ++i) {
                    const uint32_t col = tmem_base + row_off + static_cast<uint32_t>(8 * i);
                    uint32_t g0[8], u0[8], g1[8], u1[8];
                    tmem_ld_32x32b_x8(col + goff, g0);
                    tmem_ld_32x32b_x8(col + uoff, u0);
                    tmem_ld_32x32b_x8(col + 2 * R + goff, g1);
                    tmem_ld_32x32b_x8(col + 2 * R + uoff, u1);
                    tmem_ld_wait8(g0);
                    tmem_ld_wait8(u0);
                    tmem_ld_wait8(g1);
                    tmem_ld_wait8(u1);
                    if (m_lane < M) {
                        float g[8], u[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            g[c] = __uint_as_float(g0[c]) + __uint_as_float(g1[c]);
                            u[c] = __uint_as_float(u0[c]) + __uint_as_float(u1[c]);
                        }
                        uint4 h;
                        h.x = pack_bf16x2(act::gated<false>(which_act, alpha, g[0], u[0]),
                                          act::gated<false>(which_act, alpha, g[1], u[1]));
                        h.y = pack_bf16x2(act::gated<false>(which_act, alpha, g[2], u[2]),
                                          act::gated<false>(which_act, alpha, g[3], u[3]));
                        h.z = pack_bf16x2(act::gated<false>(which_act, alpha, g[4], u[4]),
                                          act::gated<false>(which_act, alpha, g[5], u[5]));
                        h.w = pack_bf16x2(act::gated<false>(which_act, alpha, g[6], u[6]),
                                          act::gated<false>(which_act, alpha, g[7], u[7]));
                        const size_t o = static_cast<size_t>(m_lane) * N + 8 * (u_begin + i);
                        *reinterpret_cast<uint4 *>(H + o) = h;
                        if (Gout) {
                            *reinterpret_cast<uint4 *>(Gout + o) =
                                make_uint4(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]),
                                           pack_bf16x2(g[4], g[5]), pack_bf16x2(g[6], g[7]));
                            *reinterpret_cast<uint4 *>(Uout + o) =
                                make_uint4(pack_bf16x2(u[0], u[1]), pack_bf16x2(u[2], u[3]),
                                           pack_bf16x2(u[4], u[5]), pack_bf16x2(u[6], u[7]));
                        }
                    }
                }
            }
            for (int i0 = 0; i0 < cnt && geo.mma_m == 64; i0 += geo.epi_units) {
                const int uc = cnt - i0 < geo.epi_units ? cnt - i0 : geo.epi_units;
                if (warp >= 2 && quad * rows_per_quad < M) {
                    for (int ii = 0; ii < uc; ++ii) {
                        const uint32_t col =
                            tmem_base + row_off + static_cast<uint32_t>(8 * (i0 + ii));
                        uint32_t g0[8], u0[8], g1[8], u1[8];
                        tmem_ld_32x32b_x8(col + goff, g0);
                        tmem_ld_32x32b_x8(col + uoff, u0);
                        tmem_ld_32x32b_x8(col + 2 * R + goff, g1);
                        tmem_ld_32x32b_x8(col + 2 * R + uoff, u1);
                        tmem_ld_wait8(g0);
                        tmem_ld_wait8(u0);
                        tmem_ld_wait8(g1);
                        tmem_ld_wait8(u1);
                        if (m_lane < M) {
                            float4 *e = reinterpret_cast<float4 *>(E + (m_lane * uc + ii) * 16);
#pragma unroll
                            for (int v = 0; v < 2; ++v) {
                                e[v] = make_float4(
                                    __uint_as_float(g0[4 * v]) + __uint_as_float(g1[4 * v]),
                                    __uint_as_float(g0[4 * v + 1]) + __uint_as_float(g1[4 * v + 1]),
                                    __uint_as_float(g0[4 * v + 2]) + __uint_as_float(g1[4 * v + 2]),
                                    __uint_as_float(g0[4 * v + 3]) + __uint_as_float(g1[4 * v + 3]));
                                e[2 + v] = make_float4(
                                    __uint_as_float(u0[4 * v]) + __uint_as_float(u1[4 * v]),
                                    __uint_as_float(u0[4 * v + 1]) + __uint_as_float(u1[4 * v + 1]),
                                    __uint_as_float(u0[4 * v + 2]) + __uint_as_float(u1[4 * v + 2]),
                                    __uint_as_float(u0[4 * v + 3]) + __uint_as_float(u1[4 * v + 3]));
                            }
                        }
                    }
                }
                named_bar_sync(1, kThreads);
                // (m, unit, column pair) items; consecutive items are
                // consecutive columns of one row of H
                const int items = M * uc * 4;
                for (int it = et; it < items; it += kThreads) {
                    const int m = it / (uc * 4);
                    const int r = it - m * uc * 4;
                    const int ii = r >> 2;
                    const int c = (r & 3) * 2;
                    const float2 g = *reinterpret_cast<const float2 *>(E + (m * uc + ii) * 16 + c);
                    const float2 u =
                        *reinterpret_cast<const float2 *>(E + (m * uc + ii) * 16 + 8 + c);
                    const size_t o = static_cast<size_t>(m) * N + 8 * (u_begin + i0 + ii) + c;
                    *reinterpret_cast<uint32_t *>(H + o) =
                        pack_bf16x2(act::gated<false>(which_act, alpha, g.x, u.x),
                                    act::gated<false>(which_act, alpha, g.y, u.y));
                    if (Gout) {
                        *reinterpret_cast<uint32_t *>(Gout + o) = pack_bf16x2(g.x, g.y);
                        *reinterpret_cast<uint32_t *>(Uout + o) = pack_bf16x2(u.x, u.y);
                    }
                }
                named_bar_sync(1, kThreads);  // E is rewritten by the next chunk
            }
        }
    }

    if (failed) atomicOr(&g_stream_tc_status, 1u);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(geo.tmem_cols));
    }
}

std::atomic<unsigned> g_attr_set_mask{0};

}  // namespace

bool stream_tc_bf16_supported(int M, int K, int N) {
    if (M < 9 || M > kStreamTcMaxM || N < 8 || N % 8 != 0) return false;
    // one CTA per SM with 16 units each always has a layout when K % 64 == 0
    return stream_geometry(M, K, 16, 220 * 1024, 2).ok;
}

cudaError_t launch_stream_tc_bf16(const void *X, const void *Wg, const void *Wu, void *H, int M,
                                  int K, int N, const Epilogue &epi, bool weights_stable,
                                  const DeviceInfo &dev, cudaStream_t stream) {
    if (N < 8 || N % 8 != 0) return cudaErrorInvalidValue;
    const StreamPlan plan = stream_plan(M, K, N, dev.sm_count);
    const StreamGeo &geo = plan.geo;
    if (!geo.ok || plan.q < 1) return cudaErrorInvalidValue;
    // 3-D views [K/64 blocks][rows][64] (rows K*2 bytes apart, blocks 128 B
    // apart) with the 128-byte swizzle: a box {64, rows, kb} lands as
    // [kb][rows][128 B].  Weight boxes are 8 q and 8 (q + 1) rows high.  The
    // pair view adds the matrix dimension (stride: the distance between the
    // buffers, from the lower one): a box {64, rows, 2, kb} lands as
    // [kb][2][rows][128 B].
    CUtensorMap tx, tg_lo, tu_lo, tg_hi, tu_hi;
    const uint64_t kblocks = static_cast<uint64_t>(geo.kblocks);
    const uint64_t row_bytes = 2ull * K;
    const uint32_t kb = static_cast<uint32_t>(geo.kb);
    const uint32_t lo = static_cast<uint32_t>(8 * plan.q);
    const uint32_t hi = static_cast<uint32_t>(8 * (plan.q + 1));
    const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_tmap_3d(&tx, X, bf, 64, M, kblocks, row_bytes, 128, 64,
                        static_cast<uint32_t>(geo.mpad), kb, sw)) {
        return cudaErrorInvalidValue;
    }
    const uintptr_t pg = reinterpret_cast<uintptr_t>(Wg), pu = reinterpret_cast<uintptr_t>(Wu);
    const int swapped = pu < pg ? 1 : 0;
    const uint64_t dist = swapped ? pg - pu : pu - pg;
    const void *w0 = swapped ? Wu : Wg;
    int pair = 0;
    if (dist != 0 && dist % 16 == 0 && dist < (1ull << 40)) {
        const uint64_t dims[4] = {64, static_cast<uint64_t>(N), 2, kblocks};
        const uint64_t strides[3] = {row_bytes, dist, 128};
        const uint32_t box_lo[4] = {64, lo, 2, kb}, box_hi[4] = {64, hi, 2, kb};
        pair = encode_tmap_4d(&tg_lo, w0, bf, dims, strides, box_lo, sw) &&
               encode_tmap_4d(&tg_hi, w0, bf, dims, strides, box_hi, sw);
        tu_lo = tg_lo;
        tu_hi = tg_hi;
    }
    if (!pair &&
        (!encode_tmap_3d(&tg_lo, Wg, bf, 64, N, kblocks, row_bytes, 128, 64, lo, kb, sw) ||
         !encode_tmap_3d(&tu_lo, Wu, bf, 64, N, kblocks, row_bytes, 128, 64, lo, kb, sw) ||
         !encode_tmap_3d(&tg_hi, Wg, bf, 64, N, kblocks, row_bytes, 128, 64, hi, kb, sw) ||
         !encode_tmap_3d(&tu_hi, Wu, bf, 64, N, kblocks, row_bytes, 128, 64, hi, kb, sw))) {
        return cudaErrorInvalidValue;
    }
    const unsigned bit = 1u << (dev.device & 31);
    if (!(g_attr_set_mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(swiglu_stream_tc_bf16_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e != cudaSuccess) return e;
        g_attr_set_mask.fetch_or(bit);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(geo.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = weights_stable ? 1 : 0;
    __nv_bfloat16 *hp = static_cast<__nv_bfloat16 *>(H);
    __nv_bfloat16 *gp = static_cast<__nv_bfloat16 *>(epi.G);
    __nv_bfloat16 *up = static_cast<__nv_bfloat16 *>(epi.U);
    const int ws = weights_stable ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, swiglu_stream_tc_bf16_kernel, tx, tg_lo, tu_lo, tg_hi,
                                       tu_hi, plan.q, pair, pair ? swapped : 0, hp, M, N, ws,
                                       epi.activation, epi.gate_multiplier, gp, up, geo, X,
                                       static_cast<uint32_t>(static_cast<size_t>(M) * K * 2));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t stream_tc_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_stream_tc_status, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_stream_tc_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
