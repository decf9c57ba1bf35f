// fk_gelu.cuh -- GELU of one fp32 value, both forms, for the elementwise
// GELU kernel and for epilogues of other kernels (LayerNorm + GELU).  The
// forms and their error analysis are described in fk_gelu.cu.
#pragma once

#include "fk.h"
#include "fk_common.cuh"

namespace fk {
namespace {

// -2 sqrt(2/pi) log2(e) and that times 0.044715, rounded once to fp32.
constexpr float kA = static_cast<float>(-2.0 * 0.79788456080286535588 * 1.44269504088896340736);
constexpr float kB = static_cast<float>(-2.0 * 0.79788456080286535588 * 1.44269504088896340736 * 0.044715);
constexpr float kRsqrt2 = 0.70710678118654752440f;

template <typename T>
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float a = x * fmaf(kB, x * x, kA);  // -2u log2(e): <= 0 for x >= 0
  const float t = Elem<T>::exp2(-fabsf(a)); // exp(-2|u|) in (0, 1]
  const float r = rcp_approx(1.0f + t);
  const float y = (a > 0.0f) ? x * t * r : x * r;
  return (x == -INFINITY) ? -0.0f : y;
}

// h = P(Z > |x|) = 0.5 erfc(|x| / sqrt 2) keeps its relative accuracy when
// tiny, so Phi(x) = 1 - h (x >= 0) or h (x < 0) is accurate to a rounding of
// Phi and y = x Phi(x) to about one ulp of y over the whole range.
__device__ __forceinline__ float gelu_erf_f(float x) {
  const float h = 0.5f * erfcf(fabsf(x) * kRsqrt2);
  const float y = x * ((x >= 0.0f) ? 1.0f - h : h);
  return (x == -INFINITY) ? -0.0f : y;
}

template <typename T, int KIND>
__device__ __forceinline__ float gelu_f(float x) {
  return KIND == FK_GELU_TANH ? gelu_tanh_f<T>(x) : gelu_erf_f(x);
}

}  // namespace
}  // namespace fk
