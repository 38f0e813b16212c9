/*
 * swiglu.h -- C ABI of the B200 (sm_100a) fused SwiGLU gate/up projection
 * library (libswiglu_b200.so).
 *
 * Operation (forward):
 *     G = X * Wg^T,  U = X * Wu^T,  H = silu(G) (.) U,  silu(x) = x*sigmoid(x)
 * computed as ONE fused op: both projections share one read of X and the
 * SiLU-and-gate step runs on the fp32 accumulators in the epilogue, so G and
 * U never reach global memory.  This is the "dual gemm with activations" of
 * Liger-Kernel issue #937 ("Another MLP implementation along with multiplier
 * support", approach 3), i.e. the "gate/up GEMM + SwiGLU in a single kernel"
 * of Liger-Kernel issue #1383 ("[RFC] Testing Methodology for FP32
 * Convergence Tests on Fused SwiGLU/dSwiGLU Kernels", Background).
 *
 * Operation (backward, elementwise "dSwiGLU", issue #1383 title/Background):
 *     dU = dH (.) silu(G),   dG = dH (.) U (.) silu'(G),
 *     silu'(x) = sigmoid(x) * (1 + x*(1 - sigmoid(x))).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to caller-owned memory on the
 *    current CUDA device, row-major and contiguous.  The library keeps no
 *    reference to them after the call returns.  Work is enqueued on `stream`
 *    (0 = legacy default stream) and runs asynchronously.
 *  - Layouts follow nn.Linear (TensorRT-LLM PR #17693 passes weight.t() to
 *    addmm and flattens rank>=3 activations to [M, in]):
 *        X [M, K], Wg [N, K], Wu [N, K], H [M, N].
 *  - Return value: SWIGLU_OK (0) or one of the SWIGLU_ERR_* codes below.
 *    Argument errors are detected on the host before anything is enqueued.
 *    A device-side wait that gave up (a bounded wait; kernels never spin
 *    forever) is reported later by swiglu_sync_status().
 *  - There is no CPU fallback and no environment-driven dispatch: routing is
 *    a pure function of (M, K, dtype), see swiglu_route_for().
 */
#ifndef SWIGLU_B200_H
#define SWIGLU_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same definition as the CUDA runtime's (driver_types.h); repeating an
 * identical typedef is legal in C11 and C++. */
typedef struct CUstream_st *cudaStream_t;

#if defined(_WIN32)
#define SWIGLU_API __declspec(dllexport)
#else
#define SWIGLU_API __attribute__((visibility("default")))
#endif

/* Element types. */
enum swiglu_dtype {
    SWIGLU_BF16 = 0, /* bf16 in/out, fp32 accumulate, bf16 RNE output       */
    SWIGLU_FP32 = 1  /* fp32 in/out, near-IEEE via 3xTF32 on tensor cores  */
};

/* Status codes. */
enum swiglu_status {
    SWIGLU_OK = 0,
    SWIGLU_ERR_NULL_POINTER = 1,     /* a required pointer is NULL          */
    SWIGLU_ERR_BAD_DIM = 2,          /* a size is negative or too large     */
    SWIGLU_ERR_MISALIGNED_DIM = 3,   /* K or N not a multiple of 8 (bf16) or
                                        4 (fp32): rows must be 16-B strided */
    SWIGLU_ERR_MISALIGNED_PTR = 4,   /* a pointer is not 16-byte aligned    */
    SWIGLU_ERR_BAD_DTYPE = 5,        /* dtype is not a swiglu_dtype         */
    SWIGLU_ERR_UNSUPPORTED_DEVICE = 6, /* current device is not sm_100      */
    SWIGLU_ERR_CUDA = 7,             /* a CUDA runtime/driver call failed   */
    SWIGLU_ERR_TIMEOUT = 8,          /* a device-side bounded wait gave up  */
    SWIGLU_ERR_OVERLAP = 9,          /* an output overlaps an input         */
    SWIGLU_ERR_NO_DEVICE = 10,       /* no CUDA device is usable            */
    SWIGLU_ERR_BAD_FLAGS = 11,       /* unknown bit in swiglu_fwd_ex flags  */
    SWIGLU_ERR_BAD_EPILOGUE = 12     /* unknown activation, non-finite gate
                                        multiplier, or only one of G/U     */
};

/* Gate activations of the epilogue variants, h = act(alpha * g) * u. */
enum swiglu_activation {
    SWIGLU_ACT_SILU = 0,      /* SwiGLU: silu(x) = x * sigmoid(x)            */
    SWIGLU_ACT_GELU_TANH = 1  /* GEGLU: x/2 (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3))) */
};

/*
 * Epilogue variant of swiglu_fwd_epilogue (Liger-Kernel issue #937: the
 * swiglu/geglu activations and the scalar gate multiplier fused into the
 * GEMM epilogue; TensorRT-LLM PR #17693: GELU(tanh) on the fp32
 * accumulator).  The multiplier scales the gate pre-activation.
 */
typedef struct swiglu_epilogue {
    int activation;        /* swiglu_activation                            */
    float gate_multiplier; /* alpha; 1.0f for none                         */
    void *G;               /* NULL, or [M, N] device output, dtype: the
                              gate projection X Wg^T (before alpha)        */
    void *U;               /* NULL, or [M, N] device output: X Wu^T.  G and
                              U are given together (training forward: the
                              backward needs them) or not at all           */
} swiglu_epilogue;

/* Flags of swiglu_fwd_ex. */
enum swiglu_flags {
    /* Wg and Wu are not written by work enqueued earlier on the stream, so
     * the decode kernel may start streaming them before that work has
     * finished (programmatic dependent launch).  X is still read, and H
     * written, only after all earlier work on the stream has completed.
     * Used by SWIGLU_ROUTE_DECODE_BF16 and SWIGLU_ROUTE_STREAM_TC_BF16,
     * ignored by the other routes. */
    SWIGLU_FLAG_WEIGHTS_STABLE = 1
};

/* Kernel routes (which kernel a swiglu_fwd call enqueues). */
enum swiglu_route {
    SWIGLU_ROUTE_NONE = 0,        /* empty problem: nothing enqueued        */
    SWIGLU_ROUTE_ZERO_K = 1,      /* K == 0: H is filled with zeros         */
    SWIGLU_ROUTE_DECODE_BF16 = 2, /* bf16, M <= 8: weight streaming with
                                     warp-level tensor-core MMA             */
    SWIGLU_ROUTE_GEMM_BF16 = 3,   /* bf16, larger M: tcgen05 dual GEMM      */
    SWIGLU_ROUTE_GEMM_TF32X3 = 4, /* fp32: 3xTF32 tcgen05 dual GEMM         */
    SWIGLU_ROUTE_BWD_GEMM_BF16 = 5, /* bf16 backward GEMM (swiglu_bwd_dx/_dw) */
    SWIGLU_ROUTE_BWD_GEMM_TF32X3 = 6, /* fp32 backward GEMM, 3xTF32         */
    SWIGLU_ROUTE_STREAM_TC_BF16 = 7 /* bf16, 9 <= M <= 128, K a multiple of
                                     64: weight streaming on tcgen05 (X the
                                     MMA's M operand, each CTA's gate and up
                                     weight rows its N operand)             */
};

/*
 * swiglu_fwd -- H = silu(X Wg^T) (.) (X Wu^T).
 *
 *  X   [M, K] device, dtype elements, 16-byte aligned.
 *  Wg  [N, K] device, dtype elements, 16-byte aligned (gate_proj.weight).
 *  Wu  [N, K] device, dtype elements, 16-byte aligned (up_proj.weight).
 *  H   [M, N] device, dtype elements, 16-byte aligned; written, never read.
 *  M, K, N >= 0.  K and N multiples of 8 (bf16) / 4 (fp32).
 *  dtype  SWIGLU_BF16 or SWIGLU_FP32.
 *
 *  M == 0 or N == 0: returns SWIGLU_OK, enqueues nothing (pointers unchecked).
 *  K == 0: H is set to +0.
 *  H must not overlap X, Wg or Wu (SWIGLU_ERR_OVERLAP).  X, Wg, Wu may alias.
 *  bf16: accumulation in fp32, SiLU and product in fp32 on the accumulators,
 *  one round-to-nearest-even to bf16; NaN/Inf propagate (no saturation).
 *  fp32: each operand is split a = hi + lo (hi, lo TF32), and the three
 *  products hi*hi + hi*lo + lo*hi are accumulated in fp32 on tensor cores.
 *  The split turns an infinite operand into NaN terms (Inf - Inf, Inf * 0),
 *  so a second, light kernel scans H and re-evaluates each NaN or infinite
 *  output in plain fp32 arithmetic: NaN and +-Inf operands give the IEEE
 *  classes of the definition, as for bf16 (finite outputs are untouched).
 *  The route (swiglu_route_for) is a pure function of M, K, N and dtype.
 *  No call allocates device memory.
 */
SWIGLU_API int swiglu_fwd(const void *X, const void *Wg, const void *Wu,
                          void *H, int64_t M, int64_t K, int64_t N, int dtype,
                          cudaStream_t stream);

/*
 * swiglu_fwd_ex -- swiglu_fwd with `flags`, a bitwise OR of swiglu_flags.
 * flags == 0 is exactly swiglu_fwd; unknown bits return
 * SWIGLU_ERR_BAD_FLAGS before anything is enqueued.
 */
SWIGLU_API int swiglu_fwd_ex(const void *X, const void *Wg, const void *Wu,
                             void *H, int64_t M, int64_t K, int64_t N,
                             int dtype, unsigned int flags,
                             cudaStream_t stream);

/*
 * swiglu_fwd_epilogue -- H = act(alpha * (X Wg^T)) (.) (X Wu^T), optionally
 * also storing G = X Wg^T and U = X Wu^T (each rounded once to dtype from
 * the fp32 accumulator).  `epi` may be NULL (SiLU, alpha = 1, no G/U, i.e.
 * swiglu_fwd_ex).  G and U follow H's rules: 16-byte aligned, no overlap
 * with any input, with H or with each other.  Same routes as swiglu_fwd.
 */
SWIGLU_API int swiglu_fwd_epilogue(const void *X, const void *Wg, const void *Wu,
                                   void *H, int64_t M, int64_t K, int64_t N,
                                   int dtype, const swiglu_epilogue *epi,
                                   unsigned int flags, cudaStream_t stream);

/*
 * swiglu_fwd_fp8 -- the forward with a quantised output: H = act(alpha G) U
 * as fp8 e4m3 with one UE8M0 scale per (1,32) block of a row (the e4m3
 * output and sf_block = (1,32) UE8M0 scale factors of TileKernels-PTO
 * PR #20, implementation notes).  For each row m and block b of columns
 * [32b, min(32b+32, N)), from the fp32 epilogue values h:
 *   amax = max |h|,  e = the smallest integer with amax <= 448 * 2^e,
 *   clamped to [-127, 127] (amax = 0: e = -127),
 *   Hs[m, b] = e + 127,   Hq[m, n] = e4m3_rne(h / 2^e)  (|h / 2^e| <= 448).
 * A block holding Inf or NaN: Hs = 0xFF and every code 0x7F (NaN).
 * Dequantised value: e4m3(Hq) * 2^(Hs - 127).
 *
 *  X, Wg, Wu  as swiglu_fwd, bf16 only (dtype argument absent).
 *  Hq   [M, N] device bytes (e4m3 codes), 16-byte aligned; N a multiple of 16.
 *  Hs   [M, ceil(N/32)] device bytes (UE8M0 codes), any alignment.
 *  epi  NULL or activation + gate multiplier; epi->G / epi->U must be NULL
 *       (SWIGLU_ERR_BAD_EPILOGUE otherwise).
 *  Every M takes the tcgen05 dual GEMM (route SWIGLU_ROUTE_GEMM_BF16).
 *  K == 0: Hq and Hs are set to 0.  Outputs must not overlap each other or
 *  an input.  Allocates no device memory.
 */
SWIGLU_API int swiglu_fwd_fp8(const void *X, const void *Wg, const void *Wu,
                              void *Hq, void *Hs, int64_t M, int64_t K,
                              int64_t N, const swiglu_epilogue *epi,
                              cudaStream_t stream);

/*
 * dswiglu_bwd -- elementwise dSwiGLU, bf16.
 *
 *  dH, G, U  [n] device bf16 inputs, 16-byte aligned.
 *  dG, dU    [n] device bf16 outputs, 16-byte aligned.
 *  n >= 0 (n == 0: no-op).  Math in fp32, one RNE rounding per output.
 *  dG may be exactly G (in place) and dU exactly U; any other overlap of an
 *  output with an input, or of dG with dU, is SWIGLU_ERR_OVERLAP.
 */
SWIGLU_API int dswiglu_bwd(const void *dH, const void *G, const void *U,
                           void *dG, void *dU, int64_t n, cudaStream_t stream);

/* dswiglu_bwd with an explicit dtype (SWIGLU_BF16 or SWIGLU_FP32). */
SWIGLU_API int dswiglu_bwd_dtype(const void *dH, const void *G, const void *U,
                                 void *dG, void *dU, int64_t n, int dtype,
                                 cudaStream_t stream);

/*
 * dswiglu_bwd_epilogue -- backward of the epilogue variants:
 *   dU = dH (.) act(alpha G),   dG = dH (.) U (.) alpha act'(alpha G).
 * activation SWIGLU_ACT_SILU with gate_multiplier 1 is dswiglu_bwd_dtype.
 * Same buffer rules as dswiglu_bwd.
 */
SWIGLU_API int dswiglu_bwd_epilogue(const void *dH, const void *G, const void *U,
                                    void *dG, void *dU, int64_t n, int dtype,
                                    int activation, float gate_multiplier,
                                    cudaStream_t stream);

/*
 * swiglu_bwd_dx -- input gradient of the projection:
 *   dX = dG Wg + dU Wu,   dX[m,k] = sum_n dG[m,n] Wg[n,k] + dU[m,n] Wu[n,k]
 * (chain rule through G = X Wg^T and U = X Wu^T; the backward half of the
 * fused MLP's forward/backward dataflow, page "[RFC] Testing Methodology for
 * FP32 Convergence Tests on Fused SwiGLU/dSwiGLU Kernels", Background).
 *
 *  dG, dU  [M, N] device, dtype elements (the outputs of dswiglu_bwd),
 *          16-byte aligned.
 *  Wg, Wu  [N, K] device, dtype elements, the forward's weights, aligned.
 *  dX      [M, K] device, dtype elements, 16-byte aligned; written only.
 *  M, K, N >= 0; K and N multiples of 8 (bf16) / 4 (fp32).
 *  dtype   SWIGLU_BF16 or SWIGLU_FP32 (else SWIGLU_ERR_BAD_DTYPE).
 *
 *  Both products accumulate in ONE fp32 accumulator (tcgen05, TMEM); bf16:
 *  dX is rounded once to bf16 (RNE); fp32: 3xTF32 products accumulated in
 *  256-deep chunks folded with round-to-nearest adds, as swiglu_fwd's fp32,
 *  and (as there) NaN or infinite outputs re-evaluated in plain fp32.
 *  M == 0 or K == 0: nothing enqueued.  N == 0: dX is set to +0.  dX must
 *  not overlap an input (SWIGLU_ERR_OVERLAP).
 *
 *  fp32 only: the output tiles beyond the last whole wave of SMs (all of
 *  them when there are fewer tiles than SMs) may be split along the
 *  reduction into parts of consecutive chunks, each folded on its own and
 *  then added in part order -- deterministic (same inputs, same bits), but
 *  those outputs are the same terms summed in another order than in
 *  swiglu_bwd_gemms.  The parts' partial tiles live in a workspace of at
 *  most (SM count) x 128 KB, allocated on `stream` for the call and freed on
 *  it afterwards (stream-ordered: cudaMallocFromPoolAsync / cudaFreeAsync,
 *  so the call can be captured in a CUDA graph) from a memory pool the
 *  library creates for the device on its first such call and keeps until
 *  the process exits; the pool keeps the memory it has mapped (the most
 *  that calls in flight at once have used: 18.5 MiB for one stream on a
 *  148-SM B200) instead of returning it at each synchronisation.
 *  SWIGLU_ERR_CUDA if the pool or the allocation fails.  bf16 allocates no
 *  device memory.
 */
SWIGLU_API int swiglu_bwd_dx(const void *dG, const void *dU, const void *Wg,
                             const void *Wu, void *dX, int64_t M, int64_t K,
                             int64_t N, int dtype, cudaStream_t stream);

/*
 * swiglu_bwd_dx_noalloc -- swiglu_bwd_dx that never allocates device memory.
 * The pages describe no such call; it exists for callers that cannot take
 * memory from the device while they run: a server or training loop that
 * reserved (nearly) all device memory for its own allocator at start-up, so
 * that the pool swiglu_bwd_dx draws its fp32 workspace from may find none
 * free, or code that forbids any allocation after initialisation.
 *
 *  Arguments, results and errors are those of swiglu_bwd_dx, and the output
 *  is bit for bit the same.  Where fp32 dX splits its tail tiles, the parts'
 *  partial tiles go to one fixed array in device memory of 18.5 MiB (the
 *  bytes of 148 partial tiles of 128 x 256 fp32, one per SM of a 148-SM
 *  B200 -- or of 74 tiles of 256 rows, one per pair of SMs -- the most any
 *  shape needs there), defined in the library: every GPU that
 *  loads the library holds it until the process exits.  A shape whose split
 *  would need more (a GPU with more SMs) returns SWIGLU_ERR_BAD_DIM before
 *  anything is enqueued.  bf16 needs no scratch and runs as swiglu_bwd_dx.
 *
 *  All calls on one GPU share the array; each call writes every part of it
 *  that it reads, so nothing needs clearing between calls, but two calls
 *  whose kernels overlap on the GPU (different streams, no ordering between
 *  them) overwrite each other's partials: order them, e.g. one stream.  The
 *  first call on each device looks up the array's device address (set-up
 *  with that device current); make that first call before any stream
 *  capture.
 */
SWIGLU_API int swiglu_bwd_dx_noalloc(const void *dG, const void *dU, const void *Wg,
                                     const void *Wu, void *dX, int64_t M, int64_t K,
                                     int64_t N, int dtype, cudaStream_t stream);

/*
 * swiglu_bwd_dw -- weight gradients of the projection:
 *   dWg = dG^T X,  dWu = dU^T X,  dWg[n,k] = sum_m dG[m,n] X[m,k]
 * (same passage as swiglu_bwd_dx).
 *
 *  dG, dU    [M, N] device, dtype elements, 16-byte aligned.
 *  X         [M, K] device, dtype elements, the forward's input, aligned.
 *  dWg, dWu  [N, K] device, dtype elements, 16-byte aligned; written, never
 *            read (not accumulated into).
 *  M, K, N >= 0; K and N multiples of 8 (bf16) / 4 (fp32).  dtype
 *  SWIGLU_BF16 or SWIGLU_FP32.
 *
 *  fp32 accumulation over all M rows in TMEM (fp32: 3xTF32, chunked as in
 *  swiglu_bwd_dx, non-finite outputs re-evaluated as there), one rounding
 *  per output.
 *  N == 0 or K == 0: nothing enqueued.  M == 0: dWg and dWu are set to +0.
 *  Outputs must not overlap each other or an input (SWIGLU_ERR_OVERLAP).
 *  Allocates no device memory.
 */
SWIGLU_API int swiglu_bwd_dw(const void *dG, const void *dU, const void *X,
                             void *dWg, void *dWu, int64_t M, int64_t K,
                             int64_t N, int dtype, cudaStream_t stream);

/*
 * swiglu_bwd_gemms -- swiglu_bwd_dx and swiglu_bwd_dw in one call:
 * dX = dG Wg + dU Wu, dWg = dG^T X, dWu = dU^T X, with the argument rules of
 * both (and dX must not overlap dWg or dWu).  The three GEMMs run as ONE
 * persistent launch whose static schedule gives every CTA its share of the
 * long dX tiles and fills with the short dW tiles, so the launch ends in one
 * balanced tail (dX alone has few tiles at small M).  The same results as
 * the two calls, bit for bit: every output is the same sum in the same order
 * whatever tile width a launch uses (the single-kind calls pick 128-, 192-
 * or 256-wide tiles by how many full waves of SMs they fill; the combined
 * launch always uses 256) -- except fp32 dX where swiglu_bwd_dx splits its
 * tail tiles (see there): never split here.  Allocates no device memory.
 */
SWIGLU_API int swiglu_bwd_gemms(const void *dG, const void *dU, const void *Wg,
                                const void *Wu, const void *X, void *dX,
                                void *dWg, void *dWu, int64_t M, int64_t K,
                                int64_t N, int dtype, cudaStream_t stream);

/* Route swiglu_fwd takes for these arguments (pure host function; returns a
 * swiglu_route, or -1 for arguments swiglu_fwd would reject). */
SWIGLU_API int swiglu_route_for(int64_t M, int64_t K, int64_t N, int dtype);

/* Route of the last swiglu_fwd* or swiglu_bwd_dx/_dw/_gemms call on this
 * host thread that returned SWIGLU_OK (SWIGLU_ROUTE_NONE before the first;
 * an empty reduction reports SWIGLU_ROUTE_ZERO_K).  Lets tests assert that
 * the fused kernel actually ran.  Kept per host thread (not per stream):
 * calls from other threads never change it, and it names the route chosen
 * on the host, not a kernel's completion. */
SWIGLU_API int swiglu_last_route(void);

/* Human-readable name of a status code (static string, never NULL). */
SWIGLU_API const char *swiglu_status_string(int status);

/*
 * Wait for `stream`, then read and clear the device status words of the
 * current device.  Returns SWIGLU_ERR_TIMEOUT if any kernel's bounded wait
 * gave up since the last call, SWIGLU_ERR_CUDA if the stream reports an
 * error, else SWIGLU_OK.
 *
 * The status words are per device and shared by every stream and host
 * thread of the process (one word per kernel family, set with an atomic OR,
 * never cleared by the kernels).  So a timeout is reported to whichever
 * swiglu_sync_status call reads the word first, whatever stream the failing
 * kernel ran on; with work on several streams, synchronise all of them (or
 * the device) before relying on which call failed.  Reading and clearing is
 * not atomic with respect to kernels still running on other streams: a wait
 * that gives up while this call runs may be reported by this call or by the
 * next one, never lost.
 */
SWIGLU_API int swiglu_sync_status(cudaStream_t stream);

/*
 * Failure-path self-test (the pages have no counterpart; it exercises this
 * library's own failure detection).  Enqueues a one-CTA kernel whose bounded
 * mbarrier wait nothing ever completes: after about a millisecond the wait
 * gives up, the kernel records it in its device status word and returns
 * normally (no trap, no fault, no hang).  The next swiglu_sync_status on the
 * stream then returns SWIGLU_ERR_TIMEOUT (and clears the word); the context
 * stays usable.  Returns SWIGLU_OK once enqueued.
 */
SWIGLU_API int swiglu_selftest_wait_timeout(cudaStream_t stream);

/*
 * Bench-only probe: stream-read `bytes` bytes from each of A and B (device,
 * 16-byte aligned, bytes a multiple of 16) into shared memory by bulk copies,
 * and write one 32-bit word per CTA to `sink` (device, at least
 * swiglu_read_floor_sink_words() words).  Measures the practical cold-read
 * floor the decode kernel is compared with (AstrAI swiglu_benchmark.md, "HBM
 * re-measurement and kernel simplification").  Launched with programmatic
 * dependent launch: it starts reading A and B while the preceding work on
 * the stream finishes (so that consecutive probes overlap as consecutive
 * weights-stable decode calls do), so A and B must not be written by earlier
 * work on the stream; `sink` is written only after that work has completed.
 */
SWIGLU_API int swiglu_read_floor(const void *A, const void *B, int64_t bytes,
                                 void *sink, cudaStream_t stream);
SWIGLU_API int64_t swiglu_read_floor_sink_words(void);

#ifdef __cplusplus
}
#endif

#endif /* SWIGLU_B200_H */
