// kernels.cuh -- internal launcher interface between the C ABI (api.cu) and
// the kernel translation units.  Every launcher only enqueues work on
// `stream` and returns the launch's cudaError_t; arguments are validated by
// the caller.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace swiglu {

// Epilogue variant of a forward call: H = act(gate_multiplier * G) * U with
// act 0 = SiLU, 1 = GELU(tanh); G and U (same dtype as H) are also stored
// when G != nullptr (then U != nullptr too).
struct Epilogue {
    int activation = 0;
    float gate_multiplier = 1.0f;
    void *G = nullptr;
    void *U = nullptr;
    // fp8 output (bf16 dual GEMM only): H is e4m3 [M, N] and `scales` the
    // UE8M0 codes [M, ceil(N/32)] of its (1,32) blocks; G/U not stored.
    void *scales = nullptr;
};

struct DeviceInfo {
    int device;
    int sm_count;
    int cc_major;
    int cc_minor;
    int max_smem_optin;  // bytes of dynamic shared memory a block may opt into
};

// bf16 forward, tcgen05 dual GEMM (any M >= 1, K >= 1, N >= 1).
cudaError_t launch_gemm_bf16(const void *X, const void *Wg, const void *Wu, void *H,
                             int M, int K, int N, const Epilogue &epi,
                             const DeviceInfo &dev, cudaStream_t stream);

// fp32 forward, 3xTF32 tcgen05 dual GEMM.
cudaError_t launch_gemm_tf32x3(const void *X, const void *Wg, const void *Wu, void *H,
                               int M, int K, int N, const Epilogue &epi,
                               const DeviceInfo &dev, cudaStream_t stream);

// bf16 forward for M <= 8: weight streaming with tensor-core dot products.
// decode_bf16_supported: whether K fits the kernel's shared-memory stages
// (a pure function of K; larger K routes to the dual GEMM).
bool decode_bf16_supported(int K);
// weights_stable: launch with programmatic dependent launch and prefetch the
// first weight stages before waiting for the preceding grid (see
// SWIGLU_FLAG_WEIGHTS_STABLE).
cudaError_t launch_decode_bf16(const void *X, const void *Wg, const void *Wu, void *H,
                               int M, int K, int N, const Epilogue &epi, bool weights_stable,
                               const DeviceInfo &dev, cudaStream_t stream);

// bf16 forward for 9 <= M <= kStreamTcMaxM: the weight stream on tcgen05
// (X as the 128-row operand, 8 Wg + 8 Wu rows as the 16-row one).
// stream_tc_bf16_supported: K a multiple of 64 and the X slices plus a
// weight ring fit shared memory (a pure function of the shape).
constexpr int kStreamTcMaxM = 128;
bool stream_tc_bf16_supported(int M, int K, int N);
cudaError_t launch_stream_tc_bf16(const void *X, const void *Wg, const void *Wu, void *H,
                                  int M, int K, int N, const Epilogue &epi, bool weights_stable,
                                  const DeviceInfo &dev, cudaStream_t stream);

// Elementwise backward of h = act(alpha g) u; dtype 0 = bf16, 1 = fp32.
cudaError_t launch_dswiglu(const void *dH, const void *G, const void *U, void *dG,
                           void *dU, int64_t n, int dtype, int activation, float alpha,
                           const DeviceInfo &dev, cudaStream_t stream);

// Backward GEMMs, bf16 (M, K, N >= 1; K, N multiples of 8):
//   dX = dG Wg + dU Wu  (one accumulator),  dWg = dG^T X,  dWu = dU^T X.
cudaError_t launch_bwd_dx_bf16(const void *dG, const void *dU, const void *Wg, const void *Wu,
                               void *dX, int M, int K, int N, const DeviceInfo &dev,
                               cudaStream_t stream);
cudaError_t launch_bwd_dw_bf16(const void *dG, const void *dU, const void *X, void *dWg,
                               void *dWu, int M, int K, int N, const DeviceInfo &dev,
                               cudaStream_t stream);
// All three bf16 backward GEMMs in one persistent launch (balanced schedule).
cudaError_t launch_bwd_all_bf16(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                const void *X, void *dX, void *dWg, void *dWu, int M, int K,
                                int N, const DeviceInfo &dev, cudaStream_t stream);
// fp32 backward GEMMs (3xTF32), same operations, K and N multiples of 4.
cudaError_t launch_bwd_dx_tf32x3(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                 void *dX, int M, int K, int N, const DeviceInfo &dev,
                                 cudaStream_t stream);
cudaError_t launch_bwd_dw_tf32x3(const void *dG, const void *dU, const void *X, void *dWg,
                                 void *dWu, int M, int K, int N, const DeviceInfo &dev,
                                 cudaStream_t stream);
// All three fp32 backward GEMMs in one persistent launch (balanced schedule).
cudaError_t launch_bwd_all_tf32x3(const void *dG, const void *dU, const void *Wg, const void *Wu,
                                  const void *X, void *dX, void *dWg, void *dWu, int M, int K,
                                  int N, const DeviceInfo &dev, cudaStream_t stream);
// After a 3xTF32 GEMM: re-evaluate every non-finite output in plain fp32
// arithmetic, so that infinite operands give the IEEE classes of the
// definition (the hi/lo split alone turns them into NaN).
cudaError_t launch_nonfinite_fwd_fp32(const void *X, const void *Wg, const void *Wu, void *H,
                                      int M, int K, int N, const Epilogue &epi,
                                      const DeviceInfo &dev, cudaStream_t stream);
cudaError_t launch_nonfinite_bwd_dx_fp32(const void *dG, const void *dU, const void *Wg,
                                         const void *Wu, void *dX, int M, int K, int N,
                                         const DeviceInfo &dev, cudaStream_t stream);
cudaError_t launch_nonfinite_bwd_dw_fp32(const void *dG, const void *dU, const void *X,
                                         void *dWg, void *dWu, int M, int K, int N,
                                         const DeviceInfo &dev, cudaStream_t stream);
// Output tile width (128, 192 or 256 columns) the backward GEMMs use for a raster
// of `row_tiles_total` 128-row tiles by `cols` columns.
int bwd_gemm_tile_n(int row_tiles_total, int cols, int sm_count, bool allow_192 = true);

// fp32 dX alone (gemm_bwd_tf32x3.cu): the tile width bn, the number of
// reduction parts of the tail tiles (0: no split) with the bytes of the
// partial tiles' workspace, and whether the pair form (256-row tiles over a
// pair of SMs) runs.
struct DxSplitPlan {
    int bn, parts;
    size_t workspace_bytes;
    bool pair;
};
DxSplitPlan dx_split_plan(int M, int K, int N, const DeviceInfo &dev);

// fp32 dX alone with the split tail's partials in a static device array
// (no allocation); *scratch_too_small is set when the plan needs more than
// the array holds.
cudaError_t launch_bwd_dx_tf32x3_static(const void *dG, const void *dU, const void *Wg,
                                        const void *Wu, void *dX, int M, int K, int N,
                                        const DeviceInfo &dev, cudaStream_t stream,
                                        bool *scratch_too_small);

// Pure streaming read of two buffers (bench-only floor probe).
int read_floor_grid(const DeviceInfo &dev);
cudaError_t launch_read_floor(const void *A, const void *B, int64_t bytes, void *sink,
                              const DeviceInfo &dev, cudaStream_t stream);

// Device status words of the GEMM kernels (bounded waits that gave up): read
// one into *host_out, reset it, and wait for the stream.
cudaError_t gemm_bf16_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);
cudaError_t gemm_tf32x3_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);

// The fp32 forward with each MMA over a pair of SMs (gemm_tf32x3_2sm.cu):
// taken where M has more than one 128-row block.
bool gemm_tf32x3_2sm_worth(int M);
cudaError_t launch_gemm_tf32x3_2sm(const void *X, const void *Wg, const void *Wu, void *H, int M,
                                   int K, int N, const Epilogue &epi, const DeviceInfo &dev,
                                   cudaStream_t stream);
cudaError_t gemm_tf32x3_2sm_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);
cudaError_t decode_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);
cudaError_t stream_tc_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);
cudaError_t gemm_bwd_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);
cudaError_t gemm_bwd_tf32x3_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);
cudaError_t selftest_status_fetch_and_clear(unsigned int *host_out, cudaStream_t stream);

// Failure-path self-test: one CTA whose bounded mbarrier wait (limit in SM
// clock cycles) never completes and gives up.
cudaError_t launch_selftest_wait(long long limit_cycles, cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no libcuda link).
bool tensor_maps_available();

}  // namespace swiglu
