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

// Exact form, x Phi(x).  h = P(Z > |x|) = 0.5 erfc(w), w = |x| / sqrt 2,
// keeps its relative accuracy when tiny, so Phi(x) = 1 - h (x >= 0) or h
// (x < 0) is accurate over the whole range.  erfc is taken in the form of
// Press et al. (Numerical Recipes, "erfcc"):
//     erfc(w) = t exp(P(t) - w^2),  t = 1 / (1 + w/2),
// with the degree-9 polynomial P fitted to the exact ln(erfc(w)/t) + w^2 on
// t in [0, 1] by memory_bound_fk_b200/fit_erfc.py (largest error of P with
// these fp32 coefficients: 1.1e-7, a relative error of erfc).  One MUFU.RCP,
// nine FMAs and one MUFU.EX2, against ~45 instructions for erfcf; P - w^2
// is a single FMA, so w^2 is not rounded on its own.  Errors: under 4e-7
// absolute on [-20, 20] for fp32, and a relative error of h below 2e-5
// where h is tiny (the fp32 rounding of the exponent, up to ~100).
template <typename T>
__device__ __forceinline__ float gelu_erf_f(float x) {
  const float w = fabsf(x) * kRsqrt2;
  const float t = rcp_approx(fmaf(0.5f, w, 1.0f));
  float p = 1.708727777e-01f;
  p = fmaf(p, t, -8.221522570e-01f);
  p = fmaf(p, t, 1.488515854e+00f);
  p = fmaf(p, t, -1.135203958e+00f);
  p = fmaf(p, t, 2.788680792e-01f);
  p = fmaf(p, t, -1.862880588e-01f);
  p = fmaf(p, t, 9.678418934e-02f);
  p = fmaf(p, t, 3.740919530e-01f);
  p = fmaf(p, t, 1.000023723e+00f);
  p = fmaf(p, t, -1.265512228e+00f);
  const float h = 0.5f * t * Elem<T>::exp2(fmaf(-w, w, p) * kLog2e);
  const float y = x * ((x >= 0.0f) ? 1.0f - h : h);
  return (x == -INFINITY) ? -0.0f : y;
}

template <typename T, int KIND>
__device__ __forceinline__ float gelu_f(float x) {
  return KIND == FK_GELU_TANH ? gelu_tanh_f<T>(x) : gelu_erf_f<T>(x);
}

}  // namespace
}  // namespace fk
