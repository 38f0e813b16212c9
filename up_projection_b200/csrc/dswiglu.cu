// dswiglu.cu -- elementwise dSwiGLU backward (the "dSwiGLU" of Liger-Kernel
// issue #1383).
//
//   dU = dH * silu(G),   dG = dH * U * silu'(G),
//   silu(g) = g s,  silu'(g) = s (1 + g (1 - s)),  s = sigmoid(g);
// and for the epilogue variants h = act(alpha g) u (GELU(tanh), a gate
// multiplier): dU = dH act(alpha G), dG = dH U alpha act'(alpha G).
//
// HBM-bound (3 loads + 2 stores per element): 128-bit vector accesses,
// L1-bypassing loads, streaming stores, a grid of a few CTAs per SM looping
// over the vectors.  The sigmoid is evaluated from t = exp(-|g|) so that both
// s and 1 - s are formed without cancellation:
//   g >= 0:  s = 1/(1+t),  1-s = t/(1+t);     g < 0:  s = t/(1+t),  1-s = 1/(1+t).
// fp32 I/O uses expf and IEEE division (a few ulp); bf16 I/O uses the fast
// hardware approximations, far below the bf16 output rounding.
#include <cuda_bf16.h>

#include "activation.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace swiglu {
namespace {

using namespace dev;

constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 8;
constexpr int kUnroll = 4;  // measured at n = 8192 * 14336: 6.15 TB/s vs 5.7 with 2

// dU = dh * act(alpha g),  dG = dh * u * alpha * act'(alpha g).  `which` is
// a compile-time constant at every call (the kernel is instantiated per
// activation), so the other activation's code folds away.
template <bool kFast>
__device__ __forceinline__ void dswiglu_elem(int which, float alpha, float dh, float g, float u,
                                             float &dg, float &du) {
    float a, da;
    act::value_and_slope<!kFast>(which, alpha * g, a, da);
    du = dh * a;
    dg = dh * u * alpha * da;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// One 16-byte vector of each operand: 8 bf16 elements.
__device__ __forceinline__ void vec_bf16(int which, float alpha, const uint4 &dh, const uint4 &g,
                                         const uint4 &u, uint4 &dg, uint4 &du) {
    const uint32_t *pdh = &dh.x, *pg = &g.x, *pu = &u.x;
    uint32_t *pdg = &dg.x, *pdu = &du.x;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float g0, u0, g1, u1;
        dswiglu_elem<true>(which, alpha, bf_lo(pdh[i]), bf_lo(pg[i]), bf_lo(pu[i]), g0, u0);
        dswiglu_elem<true>(which, alpha, bf_hi(pdh[i]), bf_hi(pg[i]), bf_hi(pu[i]), g1, u1);
        pdg[i] = pack_bf16x2(g0, g1);
        pdu[i] = pack_bf16x2(u0, u1);
    }
}

// 4 fp32 elements.
__device__ __forceinline__ void vec_f32(int which, float alpha, const uint4 &dh, const uint4 &g,
                                        const uint4 &u, uint4 &dg, uint4 &du) {
    const uint32_t *pdh = &dh.x, *pg = &g.x, *pu = &u.x;
    uint32_t *pdg = &dg.x, *pdu = &du.x;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float a, b;
        dswiglu_elem<false>(which, alpha, __uint_as_float(pdh[i]), __uint_as_float(pg[i]),
                            __uint_as_float(pu[i]), a, b);
        pdg[i] = __float_as_uint(a);
        pdu[i] = __float_as_uint(b);
    }
}

// (Three CTAs' worth of registers per SM, the occupancy the kernel has
// anyway: B200, bf16 at n = 8192 * 14336, 6.11 -> 6.35 TB/s from the code
// this bound produces; four per SM spilled and ran at 5.9.)
template <bool kBf16, int kAct>
__global__ void __launch_bounds__(kThreads, 3)
    dswiglu_kernel(const uint4 *dH, const uint4 *G, const uint4 *U, uint4 *dG, uint4 *dU,
                   int64_t nvec, const void *dH_tail, const void *G_tail, const void *U_tail,
                   void *dG_tail, void *dU_tail, int tail, float alpha) {
    constexpr int which = kAct;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < nvec; i += kUnroll * stride) {
        uint4 a[kUnroll], b[kUnroll], c[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            a[j] = ld_stream_v4(dH + i + j * stride);
            b[j] = ld_stream_v4(G + i + j * stride);
            c[j] = ld_stream_v4(U + i + j * stride);
        }
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            uint4 og, ou;
            if (kBf16) vec_bf16(which, alpha, a[j], b[j], c[j], og, ou);
            else vec_f32(which, alpha, a[j], b[j], c[j], og, ou);
            st_stream_v4(dG + i + j * stride, og);
            st_stream_v4(dU + i + j * stride, ou);
        }
    }
    for (; i < nvec; i += stride) {
        const uint4 a = ld_stream_v4(dH + i), b = ld_stream_v4(G + i), c = ld_stream_v4(U + i);
        uint4 og, ou;
        if (kBf16) vec_bf16(which, alpha, a, b, c, og, ou);
        else vec_f32(which, alpha, a, b, c, og, ou);
        st_stream_v4(dG + i, og);
        st_stream_v4(dU + i, ou);
    }
    // Elements after the last whole vector (fewer than one vector's worth).
    if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < tail) {
        const int j = threadIdx.x;
        if (kBf16) {
            const __nv_bfloat16 *pdh = static_cast<const __nv_bfloat16 *>(dH_tail);
            const __nv_bfloat16 *pg = static_cast<const __nv_bfloat16 *>(G_tail);
            const __nv_bfloat16 *pu = static_cast<const __nv_bfloat16 *>(U_tail);
            float og, ou;
            dswiglu_elem<true>(which, alpha, __bfloat162float(pdh[j]), __bfloat162float(pg[j]),
                               __bfloat162float(pu[j]), og, ou);
            static_cast<__nv_bfloat16 *>(dG_tail)[j] = __float2bfloat16_rn(og);
            static_cast<__nv_bfloat16 *>(dU_tail)[j] = __float2bfloat16_rn(ou);
        } else {
            const float *pdh = static_cast<const float *>(dH_tail);
            const float *pg = static_cast<const float *>(G_tail);
            const float *pu = static_cast<const float *>(U_tail);
            float og, ou;
            dswiglu_elem<false>(which, alpha, pdh[j], pg[j], pu[j], og, ou);
            static_cast<float *>(dG_tail)[j] = og;
            static_cast<float *>(dU_tail)[j] = ou;
        }
    }
}

}  // namespace

cudaError_t launch_dswiglu(const void *dH, const void *G, const void *U, void *dG, void *dU,
                           int64_t n, int dtype, int activation, float alpha,
                           const DeviceInfo &dev, cudaStream_t stream) {
    const int per_vec = dtype == 0 ? 8 : 4;
    const int esize = dtype == 0 ? 2 : 4;
    const int64_t nvec = n / per_vec;
    const int tail = static_cast<int>(n - nvec * per_vec);
    const int64_t off = nvec * per_vec * esize;
    const char *tdh = static_cast<const char *>(dH) + off;
    const char *tg = static_cast<const char *>(G) + off;
    const char *tu = static_cast<const char *>(U) + off;
    char *tdg = static_cast<char *>(dG) + off;
    char *tdu = static_cast<char *>(dU) + off;
    const int64_t want_blocks = (nvec + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * kBlocksPerSm;
    int grid = static_cast<int>(want_blocks < cap ? want_blocks : cap);
    if (grid < 1) grid = 1;
    const uint4 *a = static_cast<const uint4 *>(dH);
    const uint4 *b = static_cast<const uint4 *>(G);
    const uint4 *c = static_cast<const uint4 *>(U);
    uint4 *og = static_cast<uint4 *>(dG);
    uint4 *ou = static_cast<uint4 *>(dU);
    if (dtype == 0 && activation == act::kGeluTanh)
        dswiglu_kernel<true, act::kGeluTanh><<<grid, kThreads, 0, stream>>>(
            a, b, c, og, ou, nvec, tdh, tg, tu, tdg, tdu, tail, alpha);
    else if (dtype == 0)
        dswiglu_kernel<true, act::kSilu><<<grid, kThreads, 0, stream>>>(
            a, b, c, og, ou, nvec, tdh, tg, tu, tdg, tdu, tail, alpha);
    else if (activation == act::kGeluTanh)
        dswiglu_kernel<false, act::kGeluTanh><<<grid, kThreads, 0, stream>>>(
            a, b, c, og, ou, nvec, tdh, tg, tu, tdg, tdu, tail, alpha);
    else
        dswiglu_kernel<false, act::kSilu><<<grid, kThreads, 0, stream>>>(
            a, b, c, og, ou, nvec, tdh, tg, tu, tdg, tdu, tail, alpha);
    return cudaGetLastError();
}

}  // namespace swiglu
