// nonfinite_fp32.cu -- the IEEE classes (NaN, +-Inf) of the 3xTF32 GEMMs'
// outputs when an operand is infinite.
//
// 3xTF32 forms a product a*b as hi_a*hi_b + hi_a*lo_b + lo_a*hi_b.  For
// finite operands that is a*b to about 2^-22, but not for a = +-Inf: then
// lo_a = rna(a - hi_a) = NaN, and even with lo_a forced to 0 the term
// hi_a*lo_b would be Inf*0 = NaN whenever b is exactly a tf32 value.  IEEE
// arithmetic of the definition gives +-Inf for Inf*b with b finite and
// nonzero.  Every output a non-finite operand reaches is non-finite after the
// GEMM (a NaN or infinite term makes the accumulated sum non-finite), so one
// pass after the GEMM re-evaluates exactly the non-finite outputs: it scans
// the output (L2-resident right after the GEMM) and, for each non-finite
// element, recomputes its sums of products in plain fp32 arithmetic, whose
// NaN/Inf class is the one IEEE arithmetic of the definition gives whatever
// the summation order (NaN absorbs; infinities of both signs give NaN; a
// nonzero finite factor keeps an infinity's sign).  Finite outputs are left
// untouched, and outputs that are infinite because finite values overflowed
// come out infinite again.  When nothing is non-finite the pass is one read
// of the output.
#include <stdint.h>

#include "activation.cuh"
#include "kernels.cuh"

namespace swiglu {
namespace {

constexpr int kThreads = 256;

// Bit q set when component q of the vector is NaN or infinite.
__device__ __forceinline__ unsigned nonfinite_mask(float4 v) {
    return (isfinite(v.x) ? 0u : 1u) | (isfinite(v.y) ? 0u : 2u) | (isfinite(v.z) ? 0u : 4u) |
           (isfinite(v.w) ? 0u : 8u);
}

// sum_r a[r * as] * b[r * bs] for r < len, in fp32, ascending r; stops early
// once the sum is NaN (it stays NaN).
__device__ float strided_dot(const float *__restrict__ a, int64_t as, const float *__restrict__ b,
                             int64_t bs, int64_t len) {
    float s = 0.0f;
    for (int64_t r = 0; r < len; ++r) {
        s = __fadd_rn(s, __fmul_rn(a[r * as], b[r * bs]));
        if (s != s) break;
    }
    return s;
}

// Forward: H[m, n] = act(alpha g) u with g = X[m] . Wg[n], u = X[m] . Wu[n];
// the stored G and U of a training forward are refreshed too (a finite stored
// value is kept: it is the GEMM's more accurate sum).
__global__ void __launch_bounds__(kThreads)
    nonfinite_fwd_kernel(const float *__restrict__ X, const float *__restrict__ Wg,
                         const float *__restrict__ Wu, float *__restrict__ H,
                         float *__restrict__ G, float *__restrict__ U, int64_t M, int64_t K,
                         int64_t N, int which_act, float alpha) {
    const int64_t vecs = M * N / 4;  // N is a multiple of 4
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < vecs;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        for (unsigned bad = nonfinite_mask(reinterpret_cast<const float4 *>(H)[v]); bad;
             bad &= bad - 1) {
            const int64_t i = 4 * v + (__ffs(bad) - 1);
            const int64_t m = i / N, n = i - m * N;
            float g = G ? G[i] : __int_as_float(0x7fc00000);
            float u = U ? U[i] : __int_as_float(0x7fc00000);
            if (!isfinite(g)) g = strided_dot(X + m * K, 1, Wg + n * K, 1, K);
            if (!isfinite(u)) u = strided_dot(X + m * K, 1, Wu + n * K, 1, K);
            H[i] = act::gated<true>(which_act, alpha, g, u);
            if (G) {
                G[i] = g;
                U[i] = u;
            }
        }
    }
}

// Backward dX[m, k] = dG[m] . Wg[:, k] + dU[m] . Wu[:, k] (one sum over the
// 2N terms, in the GEMM's order: the dG half first).
__global__ void __launch_bounds__(kThreads)
    nonfinite_bwd_dx_kernel(const float *__restrict__ dG, const float *__restrict__ dU,
                            const float *__restrict__ Wg, const float *__restrict__ Wu,
                            float *__restrict__ dX, int64_t M, int64_t K, int64_t N) {
    const int64_t vecs = M * K / 4;  // K is a multiple of 4
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < vecs;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        for (unsigned bad = nonfinite_mask(reinterpret_cast<const float4 *>(dX)[v]); bad;
             bad &= bad - 1) {
            const int64_t i = 4 * v + (__ffs(bad) - 1);
            const int64_t m = i / K, k = i - m * K;
            const float a = strided_dot(dG + m * N, 1, Wg + k, K, N);
            const float b = strided_dot(dU + m * N, 1, Wu + k, K, N);
            dX[i] = __fadd_rn(a, b);
        }
    }
}

// Backward dW[n, k] = D[:, n] . X[:, k] for D = dG (into dWg) and dU (dWu).
__global__ void __launch_bounds__(kThreads)
    nonfinite_bwd_dw_kernel(const float *__restrict__ dG, const float *__restrict__ dU,
                            const float *__restrict__ X, float *__restrict__ dWg,
                            float *__restrict__ dWu, int64_t M, int64_t K, int64_t N) {
    const int64_t vecs = N * K / 4;
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < 2 * vecs;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool up = v >= vecs;
        float *W = up ? dWu : dWg;
        const float *D = up ? dU : dG;
        const int64_t w = up ? v - vecs : v;
        for (unsigned bad = nonfinite_mask(reinterpret_cast<const float4 *>(W)[w]); bad;
             bad &= bad - 1) {
            const int64_t i = 4 * w + (__ffs(bad) - 1);
            const int64_t n = i / K, k = i - n * K;
            W[i] = strided_dot(D + n, N, X + k, K, M);
        }
    }
}

int scan_grid(const DeviceInfo &dev, int64_t vecs) {
    const int64_t want = (vecs + kThreads - 1) / kThreads;
    const int64_t cap = 4LL * dev.sm_count;
    return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_nonfinite_fwd_fp32(const void *X, const void *Wg, const void *Wu, void *H,
                                      int M, int K, int N, const Epilogue &epi,
                                      const DeviceInfo &dev, cudaStream_t stream) {
    const int64_t vecs = static_cast<int64_t>(M) * N / 4;
    nonfinite_fwd_kernel<<<scan_grid(dev, vecs), kThreads, 0, stream>>>(
        static_cast<const float *>(X), static_cast<const float *>(Wg),
        static_cast<const float *>(Wu), static_cast<float *>(H), static_cast<float *>(epi.G),
        static_cast<float *>(epi.U), M, K, N, epi.activation, epi.gate_multiplier);
    return cudaGetLastError();
}

cudaError_t launch_nonfinite_bwd_dx_fp32(const void *dG, const void *dU, const void *Wg,
                                         const void *Wu, void *dX, int M, int K, int N,
                                         const DeviceInfo &dev, cudaStream_t stream) {
    const int64_t vecs = static_cast<int64_t>(M) * K / 4;
    nonfinite_bwd_dx_kernel<<<scan_grid(dev, vecs), kThreads, 0, stream>>>(
        static_cast<const float *>(dG), static_cast<const float *>(dU),
        static_cast<const float *>(Wg), static_cast<const float *>(Wu), static_cast<float *>(dX),
        M, K, N);
    return cudaGetLastError();
}

cudaError_t launch_nonfinite_bwd_dw_fp32(const void *dG, const void *dU, const void *X,
                                         void *dWg, void *dWu, int M, int K, int N,
                                         const DeviceInfo &dev, cudaStream_t stream) {
    const int64_t vecs = 2LL * N * K / 4;
    nonfinite_bwd_dw_kernel<<<scan_grid(dev, vecs), kThreads, 0, stream>>>(
        static_cast<const float *>(dG), static_cast<const float *>(dU),
        static_cast<const float *>(X), static_cast<float *>(dWg), static_cast<float *>(dWu), M,
        K, N);
    return cudaGetLastError();
}

}  // namespace swiglu
