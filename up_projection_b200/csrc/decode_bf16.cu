// decode_bf16.cu -- fused SwiGLU forward for decode-sized M (1..8), bf16.
//
// At M <= 8 the op is a pair of matrix-vector products: every byte of Wg and
// Wu is used M times, so the time is the time to stream both weight matrices
// from HBM once (AstrAI swiglu_benchmark.md, "HBM re-measurement and kernel
// simplification": the fused kernel sits on the dual-stream cold-read
// floor).  This kernel is built around that:
//
//  * a unit of work is 8 consecutive output columns n0..n0+7: 8 rows of Wg
//    and the same 8 rows of Wu;
//  * the 4 warps of a CTA split the unit's K range; each lane streams 16 B
//    (8 bf16) of one Wg row and one Wu row per 32-wide k chunk with
//    L1-bypassing 128-bit loads, keeping kPrefetch chunks in flight in
//    registers (weights never touch shared memory);
//  * the dot products run on the tensor cores as mma.sync m16n8k16: the
//    16-row A operand is [8 Wg rows; 8 Wu rows], the 8-column B operand is
//    X^T (rows of X beyond M are zero).  The k order inside each 16-wide
//    step is permuted identically for A and B (a sum does not depend on the
//    order of its terms) so that every lane feeds its A fragment directly
//    from its own 16-byte load.  The accumulator then gives each lane both
//    gate and up for (n0 + lane/4, m = 2*(lane%4) + {0,1}), so the SiLU-and-
//    gate epilogue is lane-local;
//  * the four warps' fp32 partials are summed in shared memory in a fixed
//    order (deterministic, no atomics), then h = silu(g) * u in fp32 and one
//    RNE rounding to bf16.
//
// X [M, K] is staged once per CTA in shared memory (zero padded to 8 rows and
// to a multiple of 32 columns, row pitch chosen so 8-lane phases of 16-byte
// reads hit distinct banks).  The first unit's weight loads are issued before
// X is staged, since they do not depend on it.
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"
#include "ptx.cuh"

namespace swiglu {
namespace {

using namespace dev;

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kPrefetch = 8;  // 32-wide k chunks in flight per warp
constexpr int kMaxSmem = 160 * 1024;

__host__ __device__ inline int padded_k(int K) { return (K + 31) / 32 * 32; }

__host__ __device__ inline int x_pitch_bytes(int K) {
    const int b = padded_k(K) * 2;  // a multiple of 64
    return (b % 128 == 0) ? b + 64 : b;
}

__host__ __device__ inline int decode_smem_bytes(int K) {
    return 8 * x_pitch_bytes(K) + kWarps * 32 * 4 * static_cast<int>(sizeof(float));
}

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu_mul_fast(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__global__ void __launch_bounds__(kThreads)
    swiglu_decode_bf16_kernel(const __nv_bfloat16 *__restrict__ X,
                              const __nv_bfloat16 *__restrict__ Wg,
                              const __nv_bfloat16 *__restrict__ Wu,
                              __nv_bfloat16 *__restrict__ H, int M, int K, int N) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int pitch = x_pitch_bytes(K);
    float *red = reinterpret_cast<float *>(smem + 8 * pitch);
    const uint32_t xs = smem_u32(smem);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int grp = lane >> 2;  // row of the unit (and column of B = row of X)
    const int tig = lane & 3;   // which 8-element slice of a 32-wide chunk
    const int units = N / 8;
    const int chunks = (K + 31) / 32;
    const int per_warp = (chunks + kWarps - 1) / kWarps;
    const int c_begin = min(warp * per_warp, chunks);
    const int c_end = min(c_begin + per_warp, chunks);

    uint4 wg[kPrefetch], wu[kPrefetch];

    // Issue the loads of chunk c of unit u into slot s (zeros past K).
    auto load_slot = [&](int s, int u, int c) {
        const int k = c * 32 + tig * 8;
        if (k < K) {
            const size_t off = static_cast<size_t>(u * 8 + grp) * K + k;
            wg[s] = ld_nc_stream_v4(Wg + off);
            wu[s] = ld_nc_stream_v4(Wu + off);
        } else {
            wg[s] = make_uint4(0, 0, 0, 0);
            wu[s] = make_uint4(0, 0, 0, 0);
        }
    };
    auto prologue = [&](int u) {
#pragma unroll
        for (int s = 0; s < kPrefetch; ++s)
            if (c_begin + s < c_end) load_slot(s, u, c_begin + s);
    };

    int u = blockIdx.x;
    if (u < units) prologue(u);

    // Stage X (zero rows >= M and columns >= K) while those loads fly.
    {
        const int kp = padded_k(K);
        const int vec_per_row = kp / 8;
        for (int i = threadIdx.x; i < 8 * vec_per_row; i += kThreads) {
            const int r = i / vec_per_row;
            const int k = (i - r * vec_per_row) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < M && k < K) v = *reinterpret_cast<const uint4 *>(X + static_cast<size_t>(r) * K + k);
            sts_v4(xs + r * pitch + k * 2, v);
        }
    }
    __syncthreads();

    const uint32_t x_row = xs + grp * pitch + tig * 16;
    for (; u < units; u += gridDim.x) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        for (int cb = c_begin; cb < c_end; cb += kPrefetch) {
#pragma unroll
            for (int s = 0; s < kPrefetch; ++s) {
                const int c = cb + s;
                if (c < c_end) {
                    const uint4 x = lds_v4(x_row + c * 64);
                    // k order inside each 16-wide step: lane (grp, tig) holds
                    // physical k 8*tig + {0..3} (first MMA) and 8*tig + {4..7}
                    // (second MMA) of the chunk, for A and B alike.
                    mma_m16n8k16_bf16(d, wg[s].x, wu[s].x, wg[s].y, wu[s].y, x.x, x.y);
                    mma_m16n8k16_bf16(d, wg[s].z, wu[s].z, wg[s].w, wu[s].w, x.z, x.w);
                    if (c + kPrefetch < c_end) load_slot(s, u, c + kPrefetch);
                }
            }
        }
        // Cross-warp reduction in a fixed order.
        float *mine = red + (warp * 32 + lane) * 4;
        mine[0] = d[0];
        mine[1] = d[1];
        mine[2] = d[2];
        mine[3] = d[3];
        const int u_next = u + gridDim.x;
        if (u_next < units) prologue(u_next);  // registers are free again
        __syncthreads();
        if (warp == 0) {
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float *p = red + (w * 32 + lane) * 4;
                s4[0] += p[0];
                s4[1] += p[1];
                s4[2] += p[2];
                s4[3] += p[3];
            }
            // s4[0], s4[1]: gate at m = 2*tig, 2*tig+1; s4[2], s4[3]: up.
            const int n = u * 8 + grp;
            const int m0 = 2 * tig;
            if (m0 < M) H[static_cast<size_t>(m0) * N + n] = __float2bfloat16_rn(silu_mul_fast(s4[0], s4[2]));
            if (m0 + 1 < M)
                H[static_cast<size_t>(m0 + 1) * N + n] = __float2bfloat16_rn(silu_mul_fast(s4[1], s4[3]));
        }
        __syncthreads();
    }
}

std::atomic<unsigned> g_attr_set_mask{0};

}  // namespace

bool decode_bf16_supported(int K) {
    return K >= 0 && K <= (1 << 20) && decode_smem_bytes(K) <= kMaxSmem;
}

cudaError_t launch_decode_bf16(const void *X, const void *Wg, const void *Wu, void *H, int M,
                               int K, int N, const DeviceInfo &dev, cudaStream_t stream) {
    const int smem = decode_smem_bytes(K);
    const unsigned bit = 1u << (dev.device & 31);
    if (!(g_attr_set_mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(swiglu_decode_bf16_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e != cudaSuccess) return e;
        g_attr_set_mask.fetch_or(bit);
    }
    const int units = N / 8;
    int per_sm = (200 * 1024) / smem;
    per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
    const long long want = static_cast<long long>(dev.sm_count) * per_sm;
    const int grid = static_cast<int>(units < want ? units : want);
    swiglu_decode_bf16_kernel<<<grid, kThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(X), static_cast<const __nv_bfloat16 *>(Wg),
        static_cast<const __nv_bfloat16 *>(Wu), static_cast<__nv_bfloat16 *>(H), M, K, N);
    return cudaGetLastError();
}

}  // namespace swiglu
