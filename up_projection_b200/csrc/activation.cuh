// activation.cuh -- the gate activations of the fused epilogue and of the
// elementwise backward, h = act(alpha * g) * u:
//   SiLU        silu(x) = x * sigmoid(x)                   (SwiGLU)
//   GELU(tanh)  gelu(x) = x/2 * (1 + tanh(c (x + a x^3))),  (GEGLU)
//               c = sqrt(2/pi), a = 0.044715
// and their derivatives silu'(x) = s (1 + x (1 - s)), s = sigmoid(x), and
// gelu'(x) = (1 + t)/2 + x/2 (1 - t^2) c (1 + 3 a x^2), t = tanh(c (x + a x^3)).
// The variants follow Liger-Kernel issue #937 (swiglu/geglu and the gate
// multiplier) and the GELU(tanh) epilogue of TensorRT-LLM PR #17693.
//
// GELU(tanh) is evaluated in the equivalent form gelu(x) = x * sigmoid(2y),
// y = c (x + a x^3), since (1 + tanh y)/2 = sigmoid(2y); then
// gelu'(x) = s + 2 x s (1 - s) c (1 + 3 a x^2), s = sigmoid(2y).  With s and
// 1 - s both formed without cancellation this keeps the relative accuracy
// for negative x, where 1 + tanh(y) would cancel.
//
// kAccurate = false: the hardware exp and reciprocal approximations (bf16
// outputs: errors of a few fp32 ulp, far below the bf16 rounding; the IEEE
// reciprocal's range check and branch would also keep the compiler from
// interleaving neighbouring activations -- B200, batched decode at
// AstrAI-1B: 11.05 -> 10.56 us per call).  kAccurate = true: expf and IEEE
// division (fp32 outputs, a few ulp).
#pragma once

#include <cuda_runtime.h>

namespace swiglu {
namespace act {

enum : int { kSilu = 0, kGeluTanh = 1 };

constexpr float kGeluC = 0.7978845608028654f;  // sqrt(2/pi)
constexpr float kGeluA = 0.044715f;

// sigmoid(x) and 1 - sigmoid(x) from t = exp(-|x|), neither cancelling.
template <bool kAccurate>
__device__ __forceinline__ void sigmoid_pair(float x, float &s, float &oms) {
    const float t = kAccurate ? expf(-fabsf(x)) : __expf(-fabsf(x));
    const float r = kAccurate ? 1.0f / (1.0f + t) : __fdividef(1.0f, 1.0f + t);
    const float tr = t * r;
    const bool pos = x >= 0.0f;
    s = pos ? r : tr;
    oms = pos ? tr : r;
}

template <bool kAccurate>
__device__ __forceinline__ float value(int which, float x) {
    if (which == kGeluTanh) {
        float s, oms;
        sigmoid_pair<kAccurate>(2.0f * kGeluC * (x + kGeluA * x * x * x), s, oms);
        return x * s;
    }
    float s, oms;
    sigmoid_pair<kAccurate>(x, s, oms);
    return x * s;
}

// act(x) and act'(x) together.
template <bool kAccurate>
__device__ __forceinline__ void value_and_slope(int which, float x, float &a, float &da) {
    if (which == kGeluTanh) {
        float s, oms;
        sigmoid_pair<kAccurate>(2.0f * kGeluC * (x + kGeluA * x * x * x), s, oms);
        a = x * s;
        da = s + 2.0f * x * s * oms * kGeluC * (1.0f + 3.0f * kGeluA * x * x);
        return;
    }
    float s, oms;
    sigmoid_pair<kAccurate>(x, s, oms);
    a = x * s;
    da = s * (1.0f + x * oms);
}

// The forward epilogue: h = act(alpha * g) * u on the fp32 accumulators.
template <bool kAccurate>
__device__ __forceinline__ float gated(int which, float alpha, float g, float u) {
    return value<kAccurate>(which, alpha * g) * u;
}

}  // namespace act
}  // namespace swiglu
