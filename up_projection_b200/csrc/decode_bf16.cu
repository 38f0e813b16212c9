// decode_bf16.cu -- fused SwiGLU forward for decode-sized M (1..8), bf16.
//
// At M <= 8 the op is a pair of matrix-vector products: every byte of Wg and
// Wu is used at most 8 times, so the time is the time to stream both weight
// matrices from HBM once (AstrAI swiglu_benchmark.md, "HBM re-measurement
// and kernel simplification": the fused kernel sits on the dual-stream
// cold-read floor).  The kernel is built to be that stream:
//
//  * one CTA per SM; CTA b owns a contiguous, balanced range of units, a unit
//    being 8 consecutive output columns n0..n0+7 (8 rows of Wg and the same 8
//    rows of Wu).  Units of 8 rows keep the split across 148 SMs within a few
//    percent of even at the decode shapes;
//  * warp 0 (one thread) streams each unit in k-slices with ONE TMA tensor
//    copy per weight matrix per stage: a 3-D view [N][K/inner][inner] of the
//    weights lets one box cover 8 rows x kc columns (16-24 KB).  On B200 the
//    per-SM cost of a bulk copy is nearly independent of its size up to tens
//    of KB, so few large copies are what reaches HBM speed;
//  * warps 1..4 split each slice's 32-wide k chunks and run the dot products
//    on the tensor cores as mma.sync m16n8k16: A = [8 Wg rows; 8 Wu rows],
//    B = X^T (rows of X beyond M are zero).  The k order inside each 16-wide
//    step is permuted identically for A and B (a sum does not depend on the
//    order of its terms) so each lane feeds its fragments from one 16-byte
//    shared-memory read of each operand.  Each lane then holds gate and up
//    for (n0 + lane/4, m = 2*(lane%4) + {0,1}), so the SiLU-and-gate
//    epilogue is lane-local;
//  * the four warps' fp32 partials of a unit go to one of four slots in
//    shared memory, and a fifth warp sums them in a fixed order
//    (deterministic, no atomics) and runs the epilogue: h = silu(g) * u in
//    fp32, one RNE rounding to bf16.  The dot-product warps never wait for an
//    epilogue, so they release their ring stages as soon as they have read
//    them (B200, AstrAI-1B: removing the reduction and epilogue from those
//    warps altogether saved 0.84 of 9.26 us per call, LLaMA-2 7B M = 8 3.5 of
//    33.2 us -- with one of them taking each unit's epilogue in turn, that
//    warp held its next stages).
//
// X [M, K] arrives by bulk copy while the first weight slices stream.  Waits
// are bounded (ptx.cuh); a stuck pipeline sets the status word and the
// kernel drains its copies and returns.
#include <cuda_bf16.h>

#include <atomic>

#include "activation.cuh"
#include "gemm_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace swiglu {

// Status word of this translation unit's kernel (bit 0 = a wait gave up).
__device__ unsigned int g_decode_status;

namespace {

using namespace dev;
using gemm::mbar_wait_drain;

constexpr int kConsumerWarps = 4;
constexpr int kEpilogueWarp = 1 + kConsumerWarps;  // warp 5
constexpr int kThreads = 32 * (2 + kConsumerWarps);
constexpr int kRedSlots = 4;  // units whose partials may wait for the epilogue warp
constexpr int kMaxStages = 6;
constexpr int kSmemBudget = 220 * 1024;  // stages + X stage, one CTA per SM
// With programmatic dependent launch, a footprint that lets the next call's
// CTA share the SM (2 x ~100 KB) so its weight prefetch overlaps this call's
// tail -- used when it still gives >= 3 stages of >= 512 k.
constexpr int kPdlSmemBudget = 100 * 1024;
constexpr int kMaxSmem = 227 * 1024;     // B200 opt-in limit per block
// full, empty (per stage), x, x_zero, red_full, red_empty (per slot)
constexpr int kNumBars = 2 * kMaxStages + 2 + 2 * kRedSlots;
constexpr int kRedSlotBytes = kConsumerWarps * 32 * 4 * 4;
constexpr int kRedBytes = kRedSlots * kRedSlotBytes;

struct Geometry {
    int inner;    // innermost box extent (elements): largest of 256..8 dividing K
    int slices;   // k-slices per unit
    int kc;       // k elements per slice (multiple of inner)
    int stages;   // ring depth
    int kx;       // k elements per X row in shared memory (slices * kc >= K)
    int off_x, off_red, off_bar, smem;
    bool ok;
};

// `xrows` rows of X are staged: 8 (rows >= M zero-filled in shared memory),
// or M in the compact layout (rows M..7 of the MMA's B operand are zeros in
// registers), which leaves more shared memory for weight stages.
inline Geometry geometry(int K, int budget, int xrows) {
    Geometry g{};
    g.inner = 8;
    for (int c = 256; c >= 8; c >>= 1)
        if (K % c == 0) {
            g.inner = c;
            break;
        }
    g.ok = false;
    // Fewest slices that still leave room for >= 3 stages (else >= 2); prefer
    // slices that divide K exactly.
    for (int pass = 0; pass < 4 && !g.ok; ++pass) {
        const int min_stages = pass < 2 ? 3 : 2;
        const bool exact = (pass % 2) == 0;
        for (int s = 1; s <= 256; ++s) {
            const int per = (K + s - 1) / s;
            if (exact && (K % s != 0 || (K / s) % g.inner != 0)) continue;
            const int kc = (per + g.inner - 1) / g.inner * g.inner;
            if (kc / g.inner > 256) continue;
            const int stage = 32 * kc;  // 16 rows x kc bf16
            const int xbytes = 2 * xrows * s * kc;
            int st = (budget - xbytes) / stage;
            if (st > kMaxStages) st = kMaxStages;
            if (xbytes < budget && st >= min_stages) {
                g.slices = s;
                g.kc = kc;
                g.stages = st;
                g.ok = true;
                break;
            }
        }
    }
    if (!g.ok) return g;
    g.kx = g.slices * g.kc;
    g.off_x = g.stages * 32 * g.kc;
    g.off_red = g.off_x + 2 * xrows * g.kx;
    g.off_bar = g.off_red + kRedBytes;
    g.smem = g.off_bar + 8 * kNumBars + 16 + 1024;  // + alignment slack
    if (g.smem > kMaxSmem) g.ok = false;
    return g;
}

// Shared-memory budget of a launch: the small footprint only when it keeps
// three or more stages of at least 512 k.
inline int decode_budget(int K, bool weights_stable, int xrows) {
    if (weights_stable) {
        const Geometry g = geometry(K, kPdlSmemBudget, xrows);
        if (g.ok && g.stages >= 3 && g.kc >= 512) return kPdlSmemBudget;
    }
    return kSmemBudget;
}

__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


template <bool kCompactX>
__global__ void __launch_bounds__(kThreads, 2)
    swiglu_decode_bf16_kernel(const __grid_constant__ CUtensorMap tm_wg,
                              const __grid_constant__ CUtensorMap tm_wu,
                              const __nv_bfloat16 *__restrict__ X,
                              __nv_bfloat16 *__restrict__ H, int M, int K, int N,
                              int weights_stable, int which_act, float alpha,
                              __nv_bfloat16 *__restrict__ Gout,
                              __nv_bfloat16 *__restrict__ Uout, const Geometry geo) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // The tensor maps are needed first and their fetch is the longest
    // dependency of the prologue: start it before anything else.  (The
    // geometry comes precomputed from the host for the same reason.)
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tm_wg);
        tma_prefetch_desc(&tm_wu);
        // X is read only after the dependency wait below; the first CTA to
        // start brings it into L2 now (each call's X may have been evicted
        // by the weights streamed since its last use).
        if (weights_stable && blockIdx.x == 0)
            bulk_prefetch_l2(X, static_cast<uint32_t>(M * K * 2));
    }
    // Under programmatic dependent launch the next call may be scheduled as
    // soon as every CTA of this one is running: it only prefetches weights
    // until this grid has completed (griddepcontrol.wait below).
    if (weights_stable) griddep_launch_dependents();
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (sbase - raw);
    const uint32_t stage_bytes = 32u * geo.kc;
    const uint32_t xs = sbase + geo.off_x;
    const uint32_t x_pitch = 2u * geo.kx;
    float *red = reinterpret_cast<float *>(gbase + geo.off_red);
    const uint32_t bar_full = sbase + geo.off_bar;
    const uint32_t bar_empty = bar_full + 8 * kMaxStages;
    const uint32_t bar_x = bar_empty + 8 * kMaxStages;
    const uint32_t bar_xzero = bar_x + 8;
    const uint32_t bar_red_full = bar_xzero + 8;                 // [kRedSlots]
    const uint32_t bar_red_empty = bar_red_full + 8 * kRedSlots;  // [kRedSlots]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + geo.off_bar + 8 * kNumBars);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int units = N / 8;
    const int u_begin = static_cast<int>((static_cast<long long>(units) * blockIdx.x) / gridDim.x);
    const int u_end = static_cast<int>((static_cast<long long>(units) * (blockIdx.x + 1)) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < geo.stages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, kConsumerWarps);
        }
        mbar_init(bar_x, 1);
        mbar_init(bar_xzero, kConsumerWarps);
        for (int s = 0; s < kRedSlots; ++s) {
            mbar_init(bar_red_full + 8 * s, kConsumerWarps);
            mbar_init(bar_red_empty + 8 * s, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    bool failed = false;
    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- weight stream
            // X is produced by earlier work on the stream: with weights_stable
            // the first weight stages are issued before waiting for it.
            bool x_issued = false;
            auto issue_x = [&]() {
                if (weights_stable) griddep_wait();
                mbar_arrive_expect_tx(bar_x, static_cast<uint32_t>(M * K * 2));
                if (geo.kx == K) {
                    bulk_load(xs, X, static_cast<uint32_t>(M * K * 2), bar_x);
                } else {
                    for (int m = 0; m < M; ++m)
                        bulk_load(xs + m * x_pitch, X + static_cast<size_t>(m) * K,
                                  static_cast<uint32_t>(K * 2), bar_x);
                }
                x_issued = true;
            };
            if (!weights_stable) issue_x();
            const int kb_per_slice = geo.kc / geo.inner;
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int u = u_begin; u < u_end && !failed; ++u) {
                for (int j = 0; j < geo.slices; ++j) {
                    // compact layout (deeper ring): X right after the first
                    // three stages, the rest of the ring fills behind it
                    const int x_after = (kCompactX && geo.stages > 3) ? 3 : geo.stages;
                    if (!x_issued && issued >= x_after) issue_x();
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, abort_flag)) {
                        failed = true;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t st = sbase + stage * stage_bytes;
                    mbar_arrive_expect_tx(fb, stage_bytes);
                    // box: inner x (kc / inner) x 8 rows; k beyond K is zero-filled
                    tma_load_3d(&tm_wg, fb, st, 0, j * kb_per_slice, u * 8);
                    tma_load_3d(&tm_wu, fb, st + stage_bytes / 2, 0, j * kb_per_slice, u * 8);
                    ++issued;
                    if (++stage == geo.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!x_issued) issue_x();
            // Never leave while a copy issued here may still write shared memory.
            for (int s = 0; s < geo.stages; ++s) {
                if (issued > s) {
                    const long long uses = (issued - 1 - s) / geo.stages + 1;
                    mbar_wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1));
                }
            }
            mbar_wait_drain(bar_x, 0);
        }
    } else if (warp == kEpilogueWarp) {
        // --------------------------------------------- reduction + epilogue
        // Unit i's partials are in slot i mod kRedSlots; the sum runs over the
        // dot-product warps in a fixed order.
        const int grp = lane >> 2;
        const int tig = lane & 3;
        for (int u = u_begin; u < u_end; ++u) {
            const int i = u - u_begin;
            const int slot = i % kRedSlots;
            const uint32_t par = static_cast<uint32_t>((i / kRedSlots) & 1);
            if (!mbar_wait(bar_red_full + 8 * slot, par, abort_flag)) {
                failed = true;
                break;
            }
            const float *part = red + slot * (kRedSlotBytes / 4);
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float *p = part + (w * 32 + lane) * 4;
                s4[0] += p[0];
                s4[1] += p[1];
                s4[2] += p[2];
                s4[3] += p[3];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_red_empty + 8 * slot);
            // s4[0], s4[1]: gate at m = 2*tig, 2*tig+1; s4[2], s4[3]: up.
            const int n = u * 8 + grp;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int m = 2 * tig + q;
                if (m < M) {
                    const size_t o = static_cast<size_t>(m) * N + n;
                    H[o] = __float2bfloat16_rn(act::gated<false>(which_act, alpha, s4[q], s4[2 + q]));
                    if (Gout) {
                        Gout[o] = __float2bfloat16_rn(s4[q]);
                        Uout[o] = __float2bfloat16_rn(s4[2 + q]);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------ consumers
        const int cw = warp - 1;
        const int ct = threadIdx.x - 32;  // 0..127
        const int grp = lane >> 2;
        const int tig = lane & 3;
        // Zero the X stage where the copies do not write: the columns
        // [K, kx) of rows < M and (8-row layout) the rows >= M.
        {
            const int vec_per_row = static_cast<int>(x_pitch / 16);
            const int rows = kCompactX ? M : 8;
            for (int i = ct; i < rows * vec_per_row; i += 32 * kConsumerWarps) {
                const int r = i / vec_per_row;
                const int byte = (i - r * vec_per_row) * 16;
                if (r >= M || byte >= K * 2) sts_v4(xs + r * x_pitch + byte, make_uint4(0, 0, 0, 0));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_xzero);
        if (!mbar_wait(bar_xzero, 0, abort_flag) || !mbar_wait(bar_x, 0, abort_flag)) failed = true;

        const uint32_t w_pitch = 2u * geo.kc;
        const int chunks = (geo.kc + 31) / 32;
        // compact layout: lanes of X rows >= M (grp >= M) read row 0 and
        // feed zeros (the load stays unconditional, a select discards it)
        const bool x_row_live = !kCompactX || grp < M;
        const uint32_t x_lane = xs + (x_row_live ? grp : 0) * x_pitch + tig * 16;
        int stage = 0;
        uint32_t phase = 0;
        for (int u = u_begin; u < u_end && !failed; ++u) {
            float d[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < geo.slices; ++j) {
                if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) {
                    failed = true;
                    break;
                }
                const uint32_t st = sbase + stage * stage_bytes;
                const uint32_t g_row = st + grp * w_pitch + tig * 16;
                const uint32_t u_row = st + (8 + grp) * w_pitch + tig * 16;
                const uint32_t x_row = x_lane + j * geo.kc * 2;
#pragma unroll 2
                for (int c = cw; c < chunks; c += kConsumerWarps) {
                    uint4 wg = make_uint4(0, 0, 0, 0), wu = wg, x = wg;
                    if (c * 32 + tig * 8 < geo.kc) {  // only a kc not divisible by 32 fails
                        wg = lds_v4(g_row + c * 64);
                        wu = lds_v4(u_row + c * 64);
                        if constexpr (kCompactX) {
                            const uint4 xv = lds_v4(x_row + c * 64);
                            x = x_row_live ? xv : x;
                        } else {
                            x = lds_v4(x_row + c * 64);
                        }
                    }
                    // lane (grp, tig) holds physical k 8*tig + {0..3} of the
                    // chunk for the first MMA and 8*tig + {4..7} for the
                    // second, in A and B alike; the two go to independent
                    // accumulators d and d1, so that consecutive MMAs do not
                    // wait on each other (summed once per unit)
                    mma_m16n8k16_bf16(d, wg.x, wu.x, wg.y, wu.y, x.x, x.y);
                    mma_m16n8k16_bf16(d1, wg.z, wu.z, wg.w, wu.w, x.z, x.w);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
                if (++stage == geo.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (failed) break;
            // Hand the partials to the epilogue warp: slot i mod kRedSlots,
            // free once the epilogue warp has read its previous use.
            const int i = u - u_begin;
            const int slot = i % kRedSlots;
            if (i >= kRedSlots &&
                !mbar_wait(bar_red_empty + 8 * slot,
                           static_cast<uint32_t>(((i / kRedSlots) & 1) ^ 1), abort_flag)) {
                failed = true;
                break;
            }
            float *mine = red + slot * (kRedSlotBytes / 4) + (cw * 32 + lane) * 4;
            mine[0] = d[0] + d1[0];
            mine[1] = d[1] + d1[1];
            mine[2] = d[2] + d1[2];
            mine[3] = d[3] + d1[3];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_red_full + 8 * slot);
        }
    }
    if (failed) atomicOr(&g_decode_status, 1u);
}

std::atomic<unsigned> g_attr_set_mask[2];

}  // namespace

bool decode_bf16_supported(int K) {
    if (K < 8 || K % 8 != 0 || K > (1 << 16)) return false;
    return geometry(K, kSmemBudget, 8).ok;
}

cudaError_t launch_decode_bf16(const void *X, const void *Wg, const void *Wu, void *H, int M,
                               int K, int N, const Epilogue &epi, bool weights_stable,
                               const DeviceInfo &dev, cudaStream_t stream) {
    int budget = decode_budget(K, weights_stable, 8);
    Geometry geo = geometry(K, budget, 8);
    // When the 8-row X stage rules out the overlapped two-CTAs-per-SM launch
    // (large K), staging only the M rows of X may fit it.
    bool compact = false;
    if (weights_stable && M < 8 && budget != kPdlSmemBudget &&
        decode_budget(K, true, M) == kPdlSmemBudget) {
        compact = true;
        budget = kPdlSmemBudget;
        geo = geometry(K, budget, M);
    }
    if (!geo.ok) return cudaErrorInvalidValue;
    // 3-D view of each weight matrix: [N rows][K / inner blocks][inner]; a box
    // is inner x (kc / inner) x 8 rows.
    CUtensorMap tg, tu;
    const uint64_t blocks = static_cast<uint64_t>(K / geo.inner);
    const uint32_t kb = static_cast<uint32_t>(geo.kc / geo.inner);
    if (!encode_tmap_3d(&tg, Wg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, geo.inner, blocks, N,
                        2ull * geo.inner, 2ull * K, geo.inner, kb, 8) ||
        !encode_tmap_3d(&tu, Wu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, geo.inner, blocks, N,
                        2ull * geo.inner, 2ull * K, geo.inner, kb, 8)) {
        return cudaErrorInvalidValue;
    }
    auto kernel = compact ? swiglu_decode_bf16_kernel<true> : swiglu_decode_bf16_kernel<false>;
    const unsigned bit = 1u << (dev.device & 31);
    std::atomic<unsigned> &mask = g_attr_set_mask[compact ? 1 : 0];
    if (!(mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kMaxSmem);
        if (e != cudaSuccess) return e;
        mask.fetch_or(bit);
    }
    // The small footprint fits two CTAs per SM: launch two per SM so each SM
    // keeps twice the bytes in flight (and the next call's CTAs take over SMs
    // as this call's CTAs finish).
    const int per_sm = (budget == kPdlSmemBudget) ? 2 : 1;
    const int units = N / 8;
    const int want = dev.sm_count * per_sm;
    const int grid = units < want ? units : want;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(geo.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = weights_stable ? 1 : 0;
    const __nv_bfloat16 *xp = static_cast<const __nv_bfloat16 *>(X);
    __nv_bfloat16 *hp = static_cast<__nv_bfloat16 *>(H);
    const int ws = weights_stable ? 1 : 0;
    const int which_act = epi.activation;
    const float alpha = epi.gate_multiplier;
    __nv_bfloat16 *gp = static_cast<__nv_bfloat16 *>(epi.G);
    __nv_bfloat16 *up = static_cast<__nv_bfloat16 *>(epi.U);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tg, tu, xp, hp, M, K, N, ws, which_act, alpha,
                                       gp, up, geo);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t decode_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(host_out, g_decode_status, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_decode_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

}  // namespace swiglu
