/*
 * swiglu_oracle.c -- plain fp64 CPU oracle for the fused SwiGLU gate/up
 * projection and its elementwise dSwiGLU backward.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library it checks.
 *
 * What it computes (all arithmetic in IEEE double, no fast-math):
 *
 *   G[m,n] = sum_k X[m,k] * Wg[n,k]      (ascending k)
 *   U[m,n] = sum_k X[m,k] * Wu[n,k]      (ascending k)
 *   H[m,n] = silu(G[m,n]) * U[m,n],  silu(x) = x * sigmoid(x)
 *
 * Sources:
 *  - The operation is the "dual gemm with activations" of Liger-Kernel issue
 *    #937 ("Another MLP implementation along with multiplier support",
 *    approach 3): one op takes x, gate_proj.weight and up_proj.weight and
 *    returns act(x Wg^T) * (x Wu^T).  The weights are nn.Linear weights,
 *    stored [out, in] = [N, K] row-major (same issue, the MLP code quoted in
 *    the TL;DR; and TensorRT-LLM PR #17693, which passes weight.t() to addmm).
 *  - The activation on the gate is SiLU, as in LigerSiLUMulFunction(gate,
 *    up) quoted in the TL;DR of issue #937, and the backward is the
 *    "dSwiGLU" named in the title and Background of Liger-Kernel issue #1383.
 *  - Inputs are [M, in] after flattening, per TensorRT-LLM PR #17693
 *    (description of _fused_up_proj_gelu).
 *  - The fused epilogue applies the activation to the un-rounded accumulator
 *    (TensorRT-LLM PR #17693, the numerics note of the follow-up commit that
 *    gates the GELU epilogue): the oracle therefore keeps G and U in double
 *    and never rounds them before the activation.
 *
 * The pages never write the SiLU or its derivative out; the oracle uses the
 * textbook definitions: sigmoid(x) = 1/(1+exp(-x)), silu(x) = x*sigmoid(x),
 * silu'(x) = sigmoid(x) * (1 + x*(1 - sigmoid(x))).
 *
 * Epilogue variants (the _act entry points): h = act(alpha * g) * u with
 * act = SiLU or GELU(tanh) and alpha the scalar gate multiplier; the plain
 * entry points are act = SiLU, alpha = 1.
 *
 * bf16 inputs arrive as their 16-bit patterns and are decoded here by a bit
 * shift into the top half of an IEEE float (exact), then widened to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ---- scalar definitions ------------------------------------------------ */

ORACLE_API double oracle_sigmoid(double x)
{
    /* Two algebraically equal forms; the branch only avoids exp overflow. */
    if (x >= 0.0) {
        return 1.0 / (1.0 + exp(-x));
    } else {
        double e = exp(x);
        return e / (1.0 + e);
    }
}

ORACLE_API double oracle_silu(double x)
{
    return x * oracle_sigmoid(x);
}

ORACLE_API double oracle_dsilu(double x)
{
    double s = oracle_sigmoid(x);
    return s * (1.0 + x * (1.0 - s));
}

/*
 * GELU with the tanh approximation, the "GELU(tanh)" of the GEGLU variant
 * (TensorRT-LLM PR #17693 fuses GELU(tanh) into the up projection; Liger-
 * Kernel issue #937 lists swiglu/geglu): gelu(x) = x/2 (1 + tanh(y)),
 * y = c (x + a x^3), c = sqrt(2/pi), a = 0.044715.
 *
 * Evaluated through the exact identities 1 + tanh(y) = 2 sigmoid(2y) and
 * 1 - tanh(y)^2 = 4 sigmoid(2y) sigmoid(-2y): the same function, without
 * the cancellation of 1 + tanh(y) for negative y (in double, tanh(y) rounds
 * to -1 below y = -19, where gelu(x) ~ x e^(2y) would come out as 0, and
 * loses ~13 bits already at y = -15).  Derivative by differentiation:
 * gelu'(x) = s + 2 x s (1 - s) y',  s = sigmoid(2y),  y' = c (1 + 3 a x^2).
 */
#define ORACLE_GELU_C 0.79788456080286535587989211986876 /* sqrt(2/pi) */
#define ORACLE_GELU_A 0.044715

ORACLE_API double oracle_gelu_tanh(double x)
{
    double y = ORACLE_GELU_C * (x + ORACLE_GELU_A * x * x * x);
    return x * oracle_sigmoid(2.0 * y);
}

ORACLE_API double oracle_dgelu_tanh(double x)
{
    double y = ORACLE_GELU_C * (x + ORACLE_GELU_A * x * x * x);
    double s = oracle_sigmoid(2.0 * y);
    double oms = oracle_sigmoid(-2.0 * y);
    double dy = ORACLE_GELU_C * (1.0 + 3.0 * ORACLE_GELU_A * x * x);
    return s + 2.0 * x * s * oms * dy;
}

/* Activation codes: 0 = SiLU, 1 = GELU(tanh). */
ORACLE_API double oracle_act(double x, int act)
{
    return act == 1 ? oracle_gelu_tanh(x) : oracle_silu(x);
}

ORACLE_API double oracle_dact(double x, int act)
{
    return act == 1 ? oracle_dgelu_tanh(x) : oracle_dsilu(x);
}

/* ---- input decoding ---------------------------------------------------- */

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

ORACLE_API void oracle_bf16_to_f64(const uint16_t *src, double *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = bf16_bits_to_double(src[i]);
}

ORACLE_API void oracle_f32_to_f64(const float *src, double *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = (double)src[i];
}

/* ---- forward on decoded (double) operands ------------------------------ */

/*
 * One output element: the two dot products over k in ascending order, then
 * the gate activation and the product.  Also returns the magnitude sums
 * sum_k |x*wg| and sum_k |x*wu| that bound the rounding error of any
 * summation order (used by the fp32-mode tolerance).
 */
/*
 * The epilogue variants: h = act(alpha * g) * u, where alpha is the scalar
 * gate multiplier of Liger-Kernel issue #937 (its "multiplier", for
 * Falcon-H1) applied to the gate pre-activation, and act is SiLU (SwiGLU)
 * or GELU(tanh) (GEGLU).  alpha = 1 and SiLU give the plain op.
 */
static void one_output(const double *x, const double *wg, const double *wu,
                       int64_t K, int act, double alpha, double *g_out,
                       double *u_out, double *h_out, double *ag_out,
                       double *au_out)
{
    double g = 0.0, u = 0.0, ag = 0.0, au = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double pg = x[k] * wg[k];
        double pu = x[k] * wu[k];
        g += pg;
        u += pu;
        ag += fabs(pg);
        au += fabs(pu);
    }
    if (g_out) *g_out = g;
    if (u_out) *u_out = u;
    if (h_out) *h_out = oracle_act(alpha * g, act) * u;
    if (ag_out) *ag_out = ag;
    if (au_out) *au_out = au;
}

/*
 * Full forward.  X [M,K], Wg/Wu [N,K], outputs [M,N]; any output pointer may
 * be NULL.  Rows of the output are independent, so they are spread over
 * OpenMP threads; each element's sum order does not depend on the thread
 * count.
 */
ORACLE_API void oracle_swiglu_fwd_act_f64(const double *X, const double *Wg,
                                          const double *Wu, int64_t M,
                                          int64_t K, int64_t N, int act,
                                          double alpha, double *G, double *U,
                                          double *H, double *AG, double *AU)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t o = m * N + n;
            one_output(X + m * K, Wg + n * K, Wu + n * K, K, act, alpha,
                       G ? G + o : 0, U ? U + o : 0, H ? H + o : 0,
                       AG ? AG + o : 0, AU ? AU + o : 0);
        }
    }
}

/* The plain op: SiLU, no gate multiplier. */
ORACLE_API void oracle_swiglu_fwd_f64(const double *X, const double *Wg,
                                      const double *Wu, int64_t M, int64_t K,
                                      int64_t N, double *G, double *U,
                                      double *H, double *AG, double *AU)
{
    oracle_swiglu_fwd_act_f64(X, Wg, Wu, M, K, N, 0, 1.0, G, U, H, AG, AU);
}

/*
 * Sampled forward: only the outputs (idx_m[i], idx_n[i]) for i < count.
 * Used to check full-size launches element by element without computing all
 * M*N outputs.
 */
ORACLE_API void oracle_swiglu_fwd_points_f64(const double *X, const double *Wg,
                                             const double *Wu, int64_t K,
                                             const int64_t *idx_m,
                                             const int64_t *idx_n,
                                             int64_t count, double *G,
                                             double *U, double *H, double *AG,
                                             double *AU)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        one_output(X + idx_m[i] * K, Wg + idx_n[i] * K, Wu + idx_n[i] * K, K,
                   0, 1.0, G ? G + i : 0, U ? U + i : 0, H ? H + i : 0,
                   AG ? AG + i : 0, AU ? AU + i : 0);
    }
}

/*
 * Sampled forward straight from the stored operands (full-size operands are
 * too large to widen to double whole): the three rows an output needs are
 * decoded into double buffers, then the same one_output() runs.
 */
typedef void (*decode_fn)(const void *src, int64_t offset, double *dst,
                          int64_t n);

static void decode_bf16_rows(const void *src, int64_t offset, double *dst,
                             int64_t n)
{
    const uint16_t *p = (const uint16_t *)src + offset;
    for (int64_t i = 0; i < n; ++i)
        dst[i] = bf16_bits_to_double(p[i]);
}

static void decode_f32_rows(const void *src, int64_t offset, double *dst,
                            int64_t n)
{
    const float *p = (const float *)src + offset;
    for (int64_t i = 0; i < n; ++i)
        dst[i] = (double)p[i];
}

static int fwd_points(decode_fn dec, const void *X, const void *Wg,
                      const void *Wu, int64_t K, const int64_t *idx_m,
                      const int64_t *idx_n, int64_t count, int act,
                      double alpha, double *G, double *U, double *H,
                      double *AG, double *AU)
{
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double *buf = (double *)malloc(sizeof(double) * 3 * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
        for (int64_t i = 0; i < count; ++i) {
            if (!buf) {
                failed = 1;
                continue;
            }
            dec(X, idx_m[i] * K, buf, K);
            dec(Wg, idx_n[i] * K, buf + K, K);
            dec(Wu, idx_n[i] * K, buf + 2 * K, K);
            one_output(buf, buf + K, buf + 2 * K, K, act, alpha, G ? G + i : 0,
                       U ? U + i : 0, H ? H + i : 0, AG ? AG + i : 0,
                       AU ? AU + i : 0);
        }
        free(buf);
    }
    return failed ? -1 : 0;
}

ORACLE_API int oracle_swiglu_fwd_points_act(int storage, const void *X,
                                            const void *Wg, const void *Wu,
                                            int64_t K, const int64_t *idx_m,
                                            const int64_t *idx_n,
                                            int64_t count, int act,
                                            double alpha, double *G,
                                            double *U, double *H, double *AG,
                                            double *AU)
{
    /* storage: 0 = bf16 bit patterns, 1 = fp32 */
    return fwd_points(storage == 0 ? decode_bf16_rows : decode_f32_rows, X, Wg,
                      Wu, K, idx_m, idx_n, count, act, alpha, G, U, H, AG, AU);
}

ORACLE_API int oracle_swiglu_fwd_points_bf16(const uint16_t *X,
                                             const uint16_t *Wg,
                                             const uint16_t *Wu, int64_t K,
                                             const int64_t *idx_m,
                                             const int64_t *idx_n,
                                             int64_t count, double *G,
                                             double *U, double *H, double *AG,
                                             double *AU)
{
    return fwd_points(decode_bf16_rows, X, Wg, Wu, K, idx_m, idx_n, count, 0,
                      1.0, G, U, H, AG, AU);
}

ORACLE_API int oracle_swiglu_fwd_points_f32(const float *X, const float *Wg,
                                            const float *Wu, int64_t K,
                                            const int64_t *idx_m,
                                            const int64_t *idx_n,
                                            int64_t count, double *G,
                                            double *U, double *H, double *AG,
                                            double *AU)
{
    return fwd_points(decode_f32_rows, X, Wg, Wu, K, idx_m, idx_n, count, 0,
                      1.0, G, U, H, AG, AU);
}

/* ---- dSwiGLU backward -------------------------------------------------- */

/*
 * Elementwise backward of h = act(alpha * g) * u with upstream gradient dh:
 *   dU = dh * act(alpha g)
 *   dG = dh * u * alpha * act'(alpha g)
 * (the "dSwiGLU" of Liger-Kernel issue #1383 for act = SiLU, alpha = 1).
 */
static void dswiglu_one(double dh, double g, double u, int act, double alpha,
                        double *dg, double *du)
{
    *du = dh * oracle_act(alpha * g, act);
    *dg = dh * u * alpha * oracle_dact(alpha * g, act);
}

/* n contiguous elements, double operands, any activation / multiplier. */
ORACLE_API void oracle_dswiglu_act_f64(const double *dH, const double *G,
                                       const double *U, int64_t n, int act,
                                       double alpha, double *dG, double *dU)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        dswiglu_one(dH[i], G[i], U[i], act, alpha, dG + i, dU + i);
}

/* The plain dSwiGLU, double operands. */
ORACLE_API void oracle_dswiglu_f64(const double *dH, const double *G,
                                   const double *U, int64_t n, double *dG,
                                   double *dU)
{
    oracle_dswiglu_act_f64(dH, G, U, n, 0, 1.0, dG, dU);
}

/* Same, straight from bf16 bit patterns (full-size n is large). */
ORACLE_API void oracle_dswiglu_bf16(const uint16_t *dH, const uint16_t *G,
                                    const uint16_t *U, int64_t n, double *dG,
                                    double *dU)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        dswiglu_one(bf16_bits_to_double(dH[i]), bf16_bits_to_double(G[i]),
                    bf16_bits_to_double(U[i]), 0, 1.0, dG + i, dU + i);
}

/* Same, fp32 operands. */
ORACLE_API void oracle_dswiglu_f32(const float *dH, const float *G,
                                   const float *U, int64_t n, double *dG,
                                   double *dU)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        dswiglu_one((double)dH[i], (double)G[i], (double)U[i], 0, 1.0, dG + i,
                    dU + i);
}

/* ---- backward GEMMs of the projection ----------------------------------- */

/*
 * With G = X Wg^T and U = X Wu^T, and dG, dU the gradients of the loss with
 * respect to G and U (the output of dSwiGLU), the chain rule gives
 *   dX[m,k]  = sum_n dG[m,n] Wg[n,k] + dU[m,n] Wu[n,k]
 *   dWg[n,k] = sum_m dG[m,n] X[m,k],   dWu[n,k] = sum_m dU[m,n] X[m,k]
 * (the backward half of the fused MLP's forward/backward dataflow, page
 * "[RFC] Testing Methodology for FP32 Convergence Tests on Fused
 * SwiGLU/dSwiGLU Kernels", Background).  Plain loops, ascending summation
 * index.
 */
ORACLE_API void oracle_bwd_dx_f64(const double *dG, const double *dU,
                                  const double *Wg, const double *Wu,
                                  int64_t M, int64_t K, int64_t N, double *dX)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                acc += dG[m * N + n] * Wg[n * K + k] + dU[m * N + n] * Wu[n * K + k];
            dX[m * K + k] = acc;
        }
    }
}

ORACLE_API void oracle_bwd_dw_f64(const double *dG, const double *dU,
                                  const double *X, int64_t M, int64_t K,
                                  int64_t N, double *dWg, double *dWu)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double ag = 0.0, au = 0.0;
            for (int64_t m = 0; m < M; ++m) {
                ag += dG[m * N + n] * X[m * K + k];
                au += dU[m * N + n] * X[m * K + k];
            }
            dWg[n * K + k] = ag;
            dWu[n * K + k] = au;
        }
    }
}

/* ---- quantised output: fp8 e4m3 with UE8M0 block scales ------------------ */

/*
 * The quantised output of the SwiGLU kernels of TileKernels-PTO PR #20
 * (implementation notes and validation: fp8 e4m3 output, UE8M0 scale
 * factors per sf_block = (1, 32), block amax, NaN-preserving casts).  The
 * page does not write the scale rule out; the reading used here: for each
 * row and each block of 32 consecutive columns (the last block may be
 * shorter),
 *   amax = max |h| over the block,
 *   e    = the smallest integer with amax <= 448 * 2^e (448 = largest finite
 *          e4m3), clamped to [-127, 127]; amax = 0 gives e = -127,
 *   scale code = e + 127 (UE8M0: an 8-bit biased power of two),
 *   q    = e4m3(h / 2^e), round to nearest, ties to even.
 * A block holding Inf or NaN gets scale code 0xFF (NaN) and NaN codes.
 *
 * e4m3 ("fn": no infinities): sign bit, 4 exponent bits (bias 7), 3
 * mantissa bits; exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is
 * NaN; the largest finite value is 1.75 * 2^8 = 448.
 */
ORACLE_API double oracle_e4m3_decode(int code)
{
    int sign = (code >> 7) & 1;
    int ef = (code >> 3) & 15;
    int mf = code & 7;
    double v;
    if (ef == 15 && mf == 7)
        return NAN;
    if (ef == 0)
        v = ldexp((double)mf / 8.0, -6);
    else
        v = ldexp(1.0 + (double)mf / 8.0, ef - 7);
    return sign ? -v : v;
}

/* Nearest e4m3 code by exhaustive search over the 127 non-negative finite
 * codes; an exact tie goes to the even code (mantissa LSB 0).  |v| > 448
 * has no finite code: NaN (the casts do not saturate). */
ORACLE_API int oracle_e4m3_encode(double v)
{
    if (isnan(v) || fabs(v) > 448.0)
        return 0x7F;
    double a = fabs(v);
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(oracle_e4m3_decode(c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (v < 0.0 || (v == 0.0 && signbit(v))) ? (best | 0x80) : best;
}

/* The UE8M0 exponent e of a block with maximum magnitude amax (finite). */
ORACLE_API int oracle_ue8m0_exponent(double amax)
{
    if (amax == 0.0)
        return -127;
    int e = -127;
    while (e < 127 && amax > 448.0 * ldexp(1.0, e))
        ++e;
    return e;
}

/* Quantise one row of n values: q[n] codes, s[ceil(n/32)] scale codes. */
ORACLE_API void oracle_quant_e4m3_row(const double *h, int64_t n, uint8_t *q, uint8_t *s)
{
    for (int64_t b = 0; b * 32 < n; ++b) {
        int64_t lo = b * 32, hi = lo + 32 < n ? lo + 32 : n;
        double amax = 0.0;
        int finite = 1;
        for (int64_t j = lo; j < hi; ++j) {
            if (!isfinite(h[j]))
                finite = 0;
            else if (fabs(h[j]) > amax)
                amax = fabs(h[j]);
        }
        if (!finite) {
            s[b] = 0xFF;
            for (int64_t j = lo; j < hi; ++j)
                q[j] = 0x7F;
            continue;
        }
        int e = oracle_ue8m0_exponent(amax);
        s[b] = (uint8_t)(e + 127);
        for (int64_t j = lo; j < hi; ++j)
            q[j] = (uint8_t)oracle_e4m3_encode(ldexp(h[j], -e));
    }
}

ORACLE_API void oracle_quant_e4m3(const double *H, int64_t M, int64_t N, uint8_t *q, uint8_t *s)
{
    int64_t nb = (N + 31) / 32;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        oracle_quant_e4m3_row(H + m * N, N, q + m * N, s + m * nb);
}

/* ---- timing support ------------------------------------------------------ */

/* Number of OpenMP threads the oracle's row loops use (n <= 0: the
 * runtime default).  The results do not depend on it: every output is
 * summed by one thread in ascending index order. */
#include <omp.h>
ORACLE_API void oracle_set_num_threads(int n)
{
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
}
