// api.cu -- the C ABI declared in include/swiglu.h: argument validation,
// routing on (M, K, dtype), launches on the caller's stream, status codes.
//
// Validation is pure host logic and runs before any CUDA call, so argument
// errors are reported identically with or without a GPU.  There is no CPU
// fallback: when no usable sm_100 device is current, calls fail with
// SWIGLU_ERR_NO_DEVICE / SWIGLU_ERR_UNSUPPORTED_DEVICE.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "kernels.cuh"
#include "swiglu.h"

namespace swiglu {
namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = (1LL << 31) - 1;  // TMA coordinates are 32-bit
constexpr int kDecodeMaxM = 8;

thread_local int t_last_route = SWIGLU_ROUTE_NONE;

std::mutex g_dev_mutex;
DeviceInfo g_dev_cache[kMaxDevices];
bool g_dev_valid[kMaxDevices];

// Current device's properties; returns a status code.
int current_device(DeviceInfo &out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        (void)cudaGetLastError();
        return SWIGLU_ERR_NO_DEVICE;
    }
    if (dev >= kMaxDevices) return SWIGLU_ERR_UNSUPPORTED_DEVICE;
    {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        if (g_dev_valid[dev]) {
            out = g_dev_cache[dev];
            return SWIGLU_OK;
        }
    }
    DeviceInfo d{};
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
        (void)cudaGetLastError();
        return SWIGLU_ERR_NO_DEVICE;
    }
    // The kernels are built for sm_100a only (tcgen05, TMEM).
    if (d.cc_major != 10 || d.cc_minor != 0) return SWIGLU_ERR_UNSUPPORTED_DEVICE;
    {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        g_dev_cache[dev] = d;
        g_dev_valid[dev] = true;
    }
    out = d;
    return SWIGLU_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, int64_t abytes, const void *b, int64_t bbytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

int elem_size(int dtype) { return dtype == SWIGLU_BF16 ? 2 : 4; }

// Shape/dtype rules of swiglu_fwd (no pointers involved).  Returns a status
// code; on success *route is the route the call takes.
int route_of_shape(int64_t M, int64_t K, int64_t N, int dtype, int *route) {
    if (dtype != SWIGLU_BF16 && dtype != SWIGLU_FP32) return SWIGLU_ERR_BAD_DTYPE;
    if (M < 0 || K < 0 || N < 0) return SWIGLU_ERR_BAD_DIM;
    if (M > kMaxDim || K > kMaxDim || N > kMaxDim) return SWIGLU_ERR_BAD_DIM;
    const int align = dtype == SWIGLU_BF16 ? 8 : 4;  // elements per 16 bytes
    if (K % align != 0 || N % align != 0) return SWIGLU_ERR_MISALIGNED_DIM;
    if (M == 0 || N == 0) *route = SWIGLU_ROUTE_NONE;
    else if (K == 0) *route = SWIGLU_ROUTE_ZERO_K;
    else if (dtype == SWIGLU_FP32) *route = SWIGLU_ROUTE_GEMM_TF32X3;
    else if (M <= kDecodeMaxM && decode_bf16_supported(static_cast<int>(K)))
        *route = SWIGLU_ROUTE_DECODE_BF16;
    else if (M <= kStreamTcMaxM &&
             stream_tc_bf16_supported(static_cast<int>(M), static_cast<int>(K), static_cast<int>(N)))
        *route = SWIGLU_ROUTE_STREAM_TC_BF16;
    else *route = SWIGLU_ROUTE_GEMM_BF16;
    return SWIGLU_OK;
}

// All argument checks of swiglu_fwd; they need no GPU.
int check_fwd(const void *X, const void *Wg, const void *Wu, const void *H, int64_t M,
              int64_t K, int64_t N, int dtype, int *route) {
    const int st = route_of_shape(M, K, N, dtype, route);
    if (st != SWIGLU_OK || *route == SWIGLU_ROUTE_NONE) return st;
    if (!H) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(H)) return SWIGLU_ERR_MISALIGNED_PTR;
    if (*route == SWIGLU_ROUTE_ZERO_K) return SWIGLU_OK;
    if (!X || !Wg || !Wu) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(X) || !aligned16(Wg) || !aligned16(Wu)) return SWIGLU_ERR_MISALIGNED_PTR;
    const int es = elem_size(dtype);
    const int64_t hb = M * N * es, xb = M * K * es, wb = N * K * es;
    if (overlaps(H, hb, X, xb) || overlaps(H, hb, Wg, wb) || overlaps(H, hb, Wu, wb))
        return SWIGLU_ERR_OVERLAP;
    return SWIGLU_OK;
}

// Epilogue checks (G/U buffers against the forward's buffers).
int check_epilogue(const swiglu_epilogue *epi, const void *X, const void *Wg, const void *Wu,
                   const void *H, int64_t M, int64_t K, int64_t N, int dtype, int route) {
    if (!epi) return SWIGLU_OK;
    if (epi->activation != SWIGLU_ACT_SILU && epi->activation != SWIGLU_ACT_GELU_TANH)
        return SWIGLU_ERR_BAD_EPILOGUE;
    if (!isfinite(epi->gate_multiplier)) return SWIGLU_ERR_BAD_EPILOGUE;
    if ((epi->G == nullptr) != (epi->U == nullptr)) return SWIGLU_ERR_BAD_EPILOGUE;
    if (!epi->G || route == SWIGLU_ROUTE_NONE) return SWIGLU_OK;
    if (!aligned16(epi->G) || !aligned16(epi->U)) return SWIGLU_ERR_MISALIGNED_PTR;
    const int es = elem_size(dtype);
    const int64_t ob = M * N * es;
    if (overlaps(epi->G, ob, epi->U, ob) || overlaps(epi->G, ob, H, ob) || overlaps(epi->U, ob, H, ob))
        return SWIGLU_ERR_OVERLAP;
    if (route != SWIGLU_ROUTE_ZERO_K) {
        const int64_t xb = M * K * es, wb = N * K * es;
        const void *outs[2] = {epi->G, epi->U};
        for (const void *o : outs)
            if (overlaps(o, ob, X, xb) || overlaps(o, ob, Wg, wb) || overlaps(o, ob, Wu, wb))
                return SWIGLU_ERR_OVERLAP;
    }
    return SWIGLU_OK;
}

int check_bwd(const void *dH, const void *G, const void *U, const void *dG, const void *dU,
              int64_t n, int dtype) {
    if (dtype != SWIGLU_BF16 && dtype != SWIGLU_FP32) return SWIGLU_ERR_BAD_DTYPE;
    if (n < 0) return SWIGLU_ERR_BAD_DIM;
    if (n == 0) return SWIGLU_OK;
    if (!dH || !G || !U || !dG || !dU) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(dH) || !aligned16(G) || !aligned16(U) || !aligned16(dG) || !aligned16(dU))
        return SWIGLU_ERR_MISALIGNED_PTR;
    const int64_t b = n * elem_size(dtype);
    // dG may be G exactly and dU may be U exactly (in place); nothing else.
    if (overlaps(dG, b, dU, b)) return SWIGLU_ERR_OVERLAP;
    if (overlaps(dG, b, dH, b)) return SWIGLU_ERR_OVERLAP;
    if (overlaps(dU, b, dH, b)) return SWIGLU_ERR_OVERLAP;
    if (dG != G && overlaps(dG, b, G, b)) return SWIGLU_ERR_OVERLAP;
    if (overlaps(dG, b, U, b)) return SWIGLU_ERR_OVERLAP;
    if (dU != U && overlaps(dU, b, U, b)) return SWIGLU_ERR_OVERLAP;
    if (overlaps(dU, b, G, b)) return SWIGLU_ERR_OVERLAP;
    return SWIGLU_OK;
}

// Shape rules shared by the backward GEMMs.
int check_bwd_shape(int64_t M, int64_t K, int64_t N, int dtype) {
    if (dtype != SWIGLU_BF16 && dtype != SWIGLU_FP32) return SWIGLU_ERR_BAD_DTYPE;
    if (M < 0 || K < 0 || N < 0) return SWIGLU_ERR_BAD_DIM;
    if (M > kMaxDim || K > kMaxDim || N > kMaxDim) return SWIGLU_ERR_BAD_DIM;
    const int align = dtype == SWIGLU_BF16 ? 8 : 4;  // elements per 16 bytes
    if (K % align != 0 || N % align != 0) return SWIGLU_ERR_MISALIGNED_DIM;
    return SWIGLU_OK;
}

// swiglu_bwd_dx: route NONE (nothing to write), ZERO_K (N == 0) or the GEMM.
int check_bwd_dx(const void *dG, const void *dU, const void *Wg, const void *Wu, const void *dX,
                 int64_t M, int64_t K, int64_t N, int dtype, int *route) {
    int st = check_bwd_shape(M, K, N, dtype);
    if (st != SWIGLU_OK) return st;
    *route = SWIGLU_ROUTE_NONE;
    if (M == 0 || K == 0) return SWIGLU_OK;
    if (!dX) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(dX)) return SWIGLU_ERR_MISALIGNED_PTR;
    *route = SWIGLU_ROUTE_ZERO_K;
    if (N == 0) return SWIGLU_OK;
    *route = dtype == SWIGLU_BF16 ? SWIGLU_ROUTE_BWD_GEMM_BF16 : SWIGLU_ROUTE_BWD_GEMM_TF32X3;
    if (!dG || !dU || !Wg || !Wu) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(dG) || !aligned16(dU) || !aligned16(Wg) || !aligned16(Wu))
        return SWIGLU_ERR_MISALIGNED_PTR;
    const int es = elem_size(dtype);
    const int64_t xb = M * K * es, gb = M * N * es, wb = N * K * es;
    if (overlaps(dX, xb, dG, gb) || overlaps(dX, xb, dU, gb) || overlaps(dX, xb, Wg, wb) ||
        overlaps(dX, xb, Wu, wb))
        return SWIGLU_ERR_OVERLAP;
    return SWIGLU_OK;
}

// swiglu_bwd_dw: route NONE, ZERO_K (M == 0) or the GEMM.
int check_bwd_dw(const void *dG, const void *dU, const void *X, const void *dWg,
                 const void *dWu, int64_t M, int64_t K, int64_t N, int dtype, int *route) {
    int st = check_bwd_shape(M, K, N, dtype);
    if (st != SWIGLU_OK) return st;
    *route = SWIGLU_ROUTE_NONE;
    if (N == 0 || K == 0) return SWIGLU_OK;
    if (!dWg || !dWu) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(dWg) || !aligned16(dWu)) return SWIGLU_ERR_MISALIGNED_PTR;
    const int es = elem_size(dtype);
    const int64_t wb = N * K * es;
    if (overlaps(dWg, wb, dWu, wb)) return SWIGLU_ERR_OVERLAP;
    *route = SWIGLU_ROUTE_ZERO_K;
    if (M == 0) return SWIGLU_OK;
    *route = dtype == SWIGLU_BF16 ? SWIGLU_ROUTE_BWD_GEMM_BF16 : SWIGLU_ROUTE_BWD_GEMM_TF32X3;
    if (!dG || !dU || !X) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(dG) || !aligned16(dU) || !aligned16(X)) return SWIGLU_ERR_MISALIGNED_PTR;
    const int64_t gb = M * N * es, xb = M * K * es;
    const void *outs[2] = {dWg, dWu};
    for (const void *o : outs) {
        if (overlaps(o, wb, dG, gb) || overlaps(o, wb, dU, gb) || overlaps(o, wb, X, xb))
            return SWIGLU_ERR_OVERLAP;
    }
    return SWIGLU_OK;
}

int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return SWIGLU_OK;
    (void)cudaGetLastError();
    return SWIGLU_ERR_CUDA;
}

}  // namespace
}  // namespace swiglu

using namespace swiglu;

extern "C" {

SWIGLU_API int swiglu_route_for(int64_t M, int64_t K, int64_t N, int dtype) {
    int route = SWIGLU_ROUTE_NONE;
    return route_of_shape(M, K, N, dtype, &route) == SWIGLU_OK ? route : -1;
}

SWIGLU_API int swiglu_fwd(const void *X, const void *Wg, const void *Wu, void *H, int64_t M,
                          int64_t K, int64_t N, int dtype, cudaStream_t stream) {
    return swiglu_fwd_ex(X, Wg, Wu, H, M, K, N, dtype, 0u, stream);
}

SWIGLU_API int swiglu_fwd_ex(const void *X, const void *Wg, const void *Wu, void *H, int64_t M,
                             int64_t K, int64_t N, int dtype, unsigned int flags,
                             cudaStream_t stream) {
    return swiglu_fwd_epilogue(X, Wg, Wu, H, M, K, N, dtype, nullptr, flags, stream);
}

SWIGLU_API int swiglu_fwd_epilogue(const void *X, const void *Wg, const void *Wu, void *H,
                                   int64_t M, int64_t K, int64_t N, int dtype,
                                   const swiglu_epilogue *epi, unsigned int flags,
                                   cudaStream_t stream) {
    if (flags & ~static_cast<unsigned int>(SWIGLU_FLAG_WEIGHTS_STABLE)) return SWIGLU_ERR_BAD_FLAGS;
    int route = SWIGLU_ROUTE_NONE;
    int st = check_fwd(X, Wg, Wu, H, M, K, N, dtype, &route);
    if (st != SWIGLU_OK) return st;
    st = check_epilogue(epi, X, Wg, Wu, H, M, K, N, dtype, route);
    if (st != SWIGLU_OK) return st;
    Epilogue ep;
    if (epi) {
        ep.activation = epi->activation;
        ep.gate_multiplier = epi->gate_multiplier;
        ep.G = epi->G;
        ep.U = epi->U;
    }
    if (route == SWIGLU_ROUTE_NONE) {
        t_last_route = route;
        return SWIGLU_OK;
    }
    DeviceInfo dev;
    st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
    cudaError_t e = cudaSuccess;
    switch (route) {
        case SWIGLU_ROUTE_ZERO_K: {
            // G = U = 0 and act(0) = 0 for both activations, so H = 0.
            const size_t bytes = static_cast<size_t>(M) * N * elem_size(dtype);
            e = cudaMemsetAsync(H, 0, bytes, stream);
            if (e == cudaSuccess && ep.G) e = cudaMemsetAsync(ep.G, 0, bytes, stream);
            if (e == cudaSuccess && ep.U) e = cudaMemsetAsync(ep.U, 0, bytes, stream);
            break;
        }
        case SWIGLU_ROUTE_DECODE_BF16:
            e = launch_decode_bf16(X, Wg, Wu, H, m, k, n, ep,
                                   (flags & SWIGLU_FLAG_WEIGHTS_STABLE) != 0, dev, stream);
            break;
        case SWIGLU_ROUTE_STREAM_TC_BF16:
            e = launch_stream_tc_bf16(X, Wg, Wu, H, m, k, n, ep,
                                      (flags & SWIGLU_FLAG_WEIGHTS_STABLE) != 0, dev, stream);
            break;
        case SWIGLU_ROUTE_GEMM_BF16:
            e = launch_gemm_bf16(X, Wg, Wu, H, m, k, n, ep, dev, stream);
            break;
        case SWIGLU_ROUTE_GEMM_TF32X3:
            // one SM per 128-row block, or (more than one block) pairs of SMs
            // sharing each MMA
            e = gemm_tf32x3_2sm_worth(m)
                    ? launch_gemm_tf32x3_2sm(X, Wg, Wu, H, m, k, n, ep, dev, stream)
                    : launch_gemm_tf32x3(X, Wg, Wu, H, m, k, n, ep, dev, stream);
            if (e == cudaSuccess) e = launch_nonfinite_fwd_fp32(X, Wg, Wu, H, m, k, n, ep, dev, stream);
            break;
        default:
            return SWIGLU_ERR_BAD_DTYPE;
    }
    st = from_cuda(e);
    if (st == SWIGLU_OK) t_last_route = route;
    return st;
}

SWIGLU_API int swiglu_fwd_fp8(const void *X, const void *Wg, const void *Wu, void *Hq, void *Hs,
                              int64_t M, int64_t K, int64_t N, const swiglu_epilogue *epi,
                              cudaStream_t stream) {
    int route = SWIGLU_ROUTE_NONE;
    int st = route_of_shape(M, K, N, SWIGLU_BF16, &route);
    if (st != SWIGLU_OK) return st;
    if (N % 16 != 0) return SWIGLU_ERR_MISALIGNED_DIM;
    if (epi) {
        if (epi->activation != SWIGLU_ACT_SILU && epi->activation != SWIGLU_ACT_GELU_TANH)
            return SWIGLU_ERR_BAD_EPILOGUE;
        if (!isfinite(epi->gate_multiplier)) return SWIGLU_ERR_BAD_EPILOGUE;
        if (epi->G || epi->U) return SWIGLU_ERR_BAD_EPILOGUE;
    }
    if (route == SWIGLU_ROUTE_NONE) {
        t_last_route = route;
        return SWIGLU_OK;
    }
    if (!Hq || !Hs) return SWIGLU_ERR_NULL_POINTER;
    if (!aligned16(Hq)) return SWIGLU_ERR_MISALIGNED_PTR;
    const int64_t qb = M * N, sb = M * ((N + 31) / 32);
    if (overlaps(Hq, qb, Hs, sb)) return SWIGLU_ERR_OVERLAP;
    if (route != SWIGLU_ROUTE_ZERO_K) {
        route = SWIGLU_ROUTE_GEMM_BF16;   // every M: the epilogue quantises
        if (!X || !Wg || !Wu) return SWIGLU_ERR_NULL_POINTER;
        if (!aligned16(X) || !aligned16(Wg) || !aligned16(Wu)) return SWIGLU_ERR_MISALIGNED_PTR;
        const int64_t xb = M * K * 2, wb = N * K * 2;
        const void *outs[2] = {Hq, Hs};
        const int64_t ob[2] = {qb, sb};
        for (int i = 0; i < 2; ++i)
            if (overlaps(outs[i], ob[i], X, xb) || overlaps(outs[i], ob[i], Wg, wb) ||
                overlaps(outs[i], ob[i], Wu, wb))
                return SWIGLU_ERR_OVERLAP;
    }
    DeviceInfo dev;
    st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    cudaError_t e;
    if (route == SWIGLU_ROUTE_ZERO_K) {
        // h = 0 everywhere: e4m3 code 0 and the scale code of amax = 0 (0).
        e = cudaMemsetAsync(Hq, 0, static_cast<size_t>(qb), stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(Hs, 0, static_cast<size_t>(sb), stream);
    } else {
        Epilogue ep;
        if (epi) {
            ep.activation = epi->activation;
            ep.gate_multiplier = epi->gate_multiplier;
        }
        ep.scales = Hs;
        e = launch_gemm_bf16(X, Wg, Wu, Hq, static_cast<int>(M), static_cast<int>(K),
                             static_cast<int>(N), ep, dev, stream);
    }
    st = from_cuda(e);
    if (st == SWIGLU_OK) t_last_route = route;
    return st;
}

SWIGLU_API int dswiglu_bwd_epilogue(const void *dH, const void *G, const void *U, void *dG,
                                    void *dU, int64_t n, int dtype, int activation,
                                    float gate_multiplier, cudaStream_t stream) {
    if (activation != SWIGLU_ACT_SILU && activation != SWIGLU_ACT_GELU_TANH)
        return SWIGLU_ERR_BAD_EPILOGUE;
    if (!isfinite(gate_multiplier)) return SWIGLU_ERR_BAD_EPILOGUE;
    int st = check_bwd(dH, G, U, dG, dU, n, dtype);
    if (st != SWIGLU_OK || n == 0) return st;
    DeviceInfo dev;
    st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    return from_cuda(launch_dswiglu(dH, G, U, dG, dU, n, dtype == SWIGLU_BF16 ? 0 : 1, activation,
                                    gate_multiplier, dev, stream));
}

SWIGLU_API int dswiglu_bwd_dtype(const void *dH, const void *G, const void *U, void *dG,
                                 void *dU, int64_t n, int dtype, cudaStream_t stream) {
    return dswiglu_bwd_epilogue(dH, G, U, dG, dU, n, dtype, SWIGLU_ACT_SILU, 1.0f, stream);
}

SWIGLU_API int dswiglu_bwd(const void *dH, const void *G, const void *U, void *dG, void *dU,
                           int64_t n, cudaStream_t stream) {
    return dswiglu_bwd_dtype(dH, G, U, dG, dU, n, SWIGLU_BF16, stream);
}

SWIGLU_API int swiglu_bwd_dx(const void *dG, const void *dU, const void *Wg, const void *Wu,
                             void *dX, int64_t M, int64_t K, int64_t N, int dtype,
                             cudaStream_t stream) {
    int route = SWIGLU_ROUTE_NONE;
    int st = check_bwd_dx(dG, dU, Wg, Wu, dX, M, K, N, dtype, &route);
    if (st != SWIGLU_OK) return st;
    if (route == SWIGLU_ROUTE_NONE) {
        t_last_route = route;
        return SWIGLU_OK;
    }
    DeviceInfo dev;
    st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    cudaError_t e;
    if (route == SWIGLU_ROUTE_ZERO_K)
        e = cudaMemsetAsync(dX, 0, static_cast<size_t>(M) * K * elem_size(dtype), stream);
    else if (route == SWIGLU_ROUTE_BWD_GEMM_BF16)
        e = launch_bwd_dx_bf16(dG, dU, Wg, Wu, dX, static_cast<int>(M), static_cast<int>(K),
                               static_cast<int>(N), dev, stream);
    else {
        const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
        e = launch_bwd_dx_tf32x3(dG, dU, Wg, Wu, dX, m, k, n, dev, stream);
        if (e == cudaSuccess) e = launch_nonfinite_bwd_dx_fp32(dG, dU, Wg, Wu, dX, m, k, n, dev, stream);
    }
    st = from_cuda(e);
    if (st == SWIGLU_OK) t_last_route = route;
    return st;
}

SWIGLU_API int swiglu_bwd_dx_noalloc(const void *dG, const void *dU, const void *Wg,
                                     const void *Wu, void *dX, int64_t M, int64_t K, int64_t N,
                                     int dtype, cudaStream_t stream) {
    int route = SWIGLU_ROUTE_NONE;
    int st = check_bwd_dx(dG, dU, Wg, Wu, dX, M, K, N, dtype, &route);
    if (st != SWIGLU_OK) return st;
    if (route == SWIGLU_ROUTE_NONE) {
        t_last_route = route;
        return SWIGLU_OK;
    }
    DeviceInfo dev;
    st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    cudaError_t e;
    if (route == SWIGLU_ROUTE_ZERO_K)
        e = cudaMemsetAsync(dX, 0, static_cast<size_t>(M) * K * elem_size(dtype), stream);
    else if (route == SWIGLU_ROUTE_BWD_GEMM_BF16)
        e = launch_bwd_dx_bf16(dG, dU, Wg, Wu, dX, static_cast<int>(M), static_cast<int>(K),
                               static_cast<int>(N), dev, stream);
    else {
        const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
        bool too_small = false;
        e = launch_bwd_dx_tf32x3_static(dG, dU, Wg, Wu, dX, m, k, n, dev, stream, &too_small);
        if (too_small) return SWIGLU_ERR_BAD_DIM;
        if (e == cudaSuccess) e = launch_nonfinite_bwd_dx_fp32(dG, dU, Wg, Wu, dX, m, k, n, dev, stream);
    }
    st = from_cuda(e);
    if (st == SWIGLU_OK) t_last_route = route;
    return st;
}

SWIGLU_API int swiglu_bwd_dw(const void *dG, const void *dU, const void *X, void *dWg,
                             void *dWu, int64_t M, int64_t K, int64_t N, int dtype,
                             cudaStream_t stream) {
    int route = SWIGLU_ROUTE_NONE;
    int st = check_bwd_dw(dG, dU, X, dWg, dWu, M, K, N, dtype, &route);
    if (st != SWIGLU_OK) return st;
    if (route == SWIGLU_ROUTE_NONE) {
        t_last_route = route;
        return SWIGLU_OK;
    }
    DeviceInfo dev;
    st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    cudaError_t e;
    if (route == SWIGLU_ROUTE_ZERO_K) {
        const size_t bytes = static_cast<size_t>(N) * K * elem_size(dtype);
        e = cudaMemsetAsync(dWg, 0, bytes, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dWu, 0, bytes, stream);
    } else if (route == SWIGLU_ROUTE_BWD_GEMM_BF16) {
        e = launch_bwd_dw_bf16(dG, dU, X, dWg, dWu, static_cast<int>(M), static_cast<int>(K),
                               static_cast<int>(N), dev, stream);
    } else {
        const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
        e = launch_bwd_dw_tf32x3(dG, dU, X, dWg, dWu, m, k, n, dev, stream);
        if (e == cudaSuccess)
            e = launch_nonfinite_bwd_dw_fp32(dG, dU, X, dWg, dWu, m, k, n, dev, stream);
    }
    st = from_cuda(e);
    if (st == SWIGLU_OK) t_last_route = route;
    return st;
}

SWIGLU_API int swiglu_bwd_gemms(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                const void *X, void *dX, void *dWg, void *dWu, int64_t M, int64_t K,
                                int64_t N, int dtype, cudaStream_t stream) {
    int rx = SWIGLU_ROUTE_NONE, rw = SWIGLU_ROUTE_NONE;
    int st = check_bwd_dx(dG, dU, Wg, Wu, dX, M, K, N, dtype, &rx);
    if (st != SWIGLU_OK) return st;
    st = check_bwd_dw(dG, dU, X, dWg, dWu, M, K, N, dtype, &rw);
    if (st != SWIGLU_OK) return st;
    if (rx != SWIGLU_ROUTE_NONE && rw != SWIGLU_ROUTE_NONE) {
        const int es = elem_size(dtype);
        const int64_t xb = M * K * es, wb = N * K * es;
        if (overlaps(dX, xb, dWg, wb) || overlaps(dX, xb, dWu, wb)) return SWIGLU_ERR_OVERLAP;
    }
    const bool gemm_x = rx == SWIGLU_ROUTE_BWD_GEMM_BF16 || rx == SWIGLU_ROUTE_BWD_GEMM_TF32X3;
    const bool gemm_w = rw == SWIGLU_ROUTE_BWD_GEMM_BF16 || rw == SWIGLU_ROUTE_BWD_GEMM_TF32X3;
    if (gemm_x && gemm_w) {
        DeviceInfo dev;
        st = current_device(dev);
        if (st != SWIGLU_OK) return st;
        const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
        cudaError_t e;
        if (dtype == SWIGLU_FP32) {
            e = launch_bwd_all_tf32x3(dG, dU, Wg, Wu, X, dX, dWg, dWu, m, k, n, dev, stream);
            if (e == cudaSuccess)
                e = launch_nonfinite_bwd_dx_fp32(dG, dU, Wg, Wu, dX, m, k, n, dev, stream);
            if (e == cudaSuccess)
                e = launch_nonfinite_bwd_dw_fp32(dG, dU, X, dWg, dWu, m, k, n, dev, stream);
        } else {
            e = launch_bwd_all_bf16(dG, dU, Wg, Wu, X, dX, dWg, dWu, m, k, n, dev, stream);
        }
        st = from_cuda(e);
        if (st == SWIGLU_OK) t_last_route = rx;
        return st;
    }
    // otherwise one call each (zero fills of empty reductions included)
    st = swiglu_bwd_dx(dG, dU, Wg, Wu, dX, M, K, N, dtype, stream);
    if (st != SWIGLU_OK) return st;
    return swiglu_bwd_dw(dG, dU, X, dWg, dWu, M, K, N, dtype, stream);
}

SWIGLU_API int swiglu_last_route(void) { return t_last_route; }

SWIGLU_API const char *swiglu_status_string(int status) {
    switch (status) {
        case SWIGLU_OK: return "ok";
        case SWIGLU_ERR_NULL_POINTER: return "null pointer";
        case SWIGLU_ERR_BAD_DIM: return "bad dimension (negative or too large)";
        case SWIGLU_ERR_MISALIGNED_DIM: return "K and N must be multiples of 16 bytes of elements";
        case SWIGLU_ERR_MISALIGNED_PTR: return "pointer not 16-byte aligned";
        case SWIGLU_ERR_BAD_DTYPE: return "unknown dtype";
        case SWIGLU_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100";
        case SWIGLU_ERR_CUDA: return "CUDA error";
        case SWIGLU_ERR_TIMEOUT: return "device-side bounded wait gave up";
        case SWIGLU_ERR_OVERLAP: return "output overlaps an input";
        case SWIGLU_ERR_NO_DEVICE: return "no usable CUDA device";
        case SWIGLU_ERR_BAD_FLAGS: return "unknown flag bit";
        case SWIGLU_ERR_BAD_EPILOGUE: return "bad epilogue (activation, multiplier or G/U pair)";
        default: return "unknown status";
    }
}

SWIGLU_API int swiglu_sync_status(cudaStream_t stream) {
    DeviceInfo dev;
    int st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return from_cuda(e);
    unsigned int w1 = 0, w2 = 0, w3 = 0, w4 = 0, w5 = 0, w6 = 0, w7 = 0, w8 = 0;
    e = gemm_bf16_status_fetch_and_clear(&w1, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = gemm_tf32x3_status_fetch_and_clear(&w2, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = decode_status_fetch_and_clear(&w3, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = gemm_bwd_status_fetch_and_clear(&w4, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = gemm_bwd_tf32x3_status_fetch_and_clear(&w5, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = selftest_status_fetch_and_clear(&w6, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = stream_tc_status_fetch_and_clear(&w7, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = gemm_tf32x3_2sm_status_fetch_and_clear(&w8, stream);
    if (e != cudaSuccess) return from_cuda(e);
    return (w1 | w2 | w3 | w4 | w5 | w6 | w7 | w8) ? SWIGLU_ERR_TIMEOUT : SWIGLU_OK;
}

SWIGLU_API int swiglu_selftest_wait_timeout(cudaStream_t stream) {
    DeviceInfo dev;
    int st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    // about one millisecond at the B200 boost clock
    return from_cuda(launch_selftest_wait(2000000LL, stream));
}

SWIGLU_API int swiglu_read_floor(const void *A, const void *B, int64_t bytes, void *sink,
                                 cudaStream_t stream) {
    if (!A || !B || !sink) return SWIGLU_ERR_NULL_POINTER;
    if (bytes < 0) return SWIGLU_ERR_BAD_DIM;
    if (bytes % 16 != 0) return SWIGLU_ERR_MISALIGNED_DIM;
    if (!aligned16(A) || !aligned16(B) || !aligned16(sink)) return SWIGLU_ERR_MISALIGNED_PTR;
    DeviceInfo dev;
    int st = current_device(dev);
    if (st != SWIGLU_OK) return st;
    if (read_floor_grid(dev) > swiglu_read_floor_sink_words()) return SWIGLU_ERR_BAD_DIM;
    return from_cuda(launch_read_floor(A, B, bytes, sink, dev, stream));
}

SWIGLU_API int64_t swiglu_read_floor_sink_words(void) { return 4096; }

}  // extern "C"
