// fk_gelu.cuh -- GELU of one fp32 value, both forms, for the elementwise
// GELU kernel and for epilogues of other kernels (LayerNorm + GELU).  The
// forms and their error analysis are described in fk_gelu.cu.
#pragma once

#include "fk.h"
#include "fk_common.cuh"
#include "fk_f32x2.cuh"

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
// The fitted P(t), by Horner's rule, for one value or a pair.
template <typename V>
__device__ __forceinline__ V erfc_poly(V t) {
  V p = splat_v<V>(1.708727777e-01f);
  p = fma_v(p, t, -8.221522570e-01f);
  p = fma_v(p, t, 1.488515854e+00f);
  p = fma_v(p, t, -1.135203958e+00f);
  p = fma_v(p, t, 2.788680792e-01f);
  p = fma_v(p, t, -1.862880588e-01f);
  p = fma_v(p, t, 9.678418934e-02f);
  p = fma_v(p, t, 3.740919530e-01f);
  p = fma_v(p, t, 1.000023723e+00f);
  p = fma_v(p, t, -1.265512228e+00f);
  return p;
}

template <typename T>
__device__ __forceinline__ float gelu_erf_f(float x) {
  const float w = fabsf(x) * kRsqrt2;
  const float t = rcp_approx(fmaf(0.5f, w, 1.0f));
  const float p = erfc_poly(t);
  const float h = 0.5f * t * Elem<T>::exp2(fmaf(-w, w, p) * kLog2e);
  const float y = x * ((x >= 0.0f) ? 1.0f - h : h);
  return (x == -INFINITY) ? -0.0f : y;
}

// The two forms on a pair of values: every lane takes the operations of the
// scalar functions above in the same order (packed fp32 arithmetic rounds
// each lane as the scalar instruction does), so the results are identical,
// with about half the arithmetic instructions.
template <typename T>
__device__ __forceinline__ float2 gelu_tanh_f2(float2 x) {
  const float2 a = mul2(x, fma2(splat2(kB), mul2(x, x), splat2(kA)));
  const float2 t = make_float2(Elem<T>::exp2(-fabsf(a.x)), Elem<T>::exp2(-fabsf(a.y)));
  const float2 s = add2(splat2(1.0f), t);
  const float2 r = make_float2(rcp_approx(s.x), rcp_approx(s.y));
  const float2 yp = mul2(mul2(x, t), r);  // x t r, for a > 0
  const float2 yn = mul2(x, r);
  float2 y = make_float2(a.x > 0.0f ? yp.x : yn.x, a.y > 0.0f ? yp.y : yn.y);
  y.x = (x.x == -INFINITY) ? -0.0f : y.x;
  y.y = (x.y == -INFINITY) ? -0.0f : y.y;
  return y;
}

template <typename T>
__device__ __forceinline__ float2 gelu_erf_f2(float2 x) {
  const float2 w = mul2(make_float2(fabsf(x.x), fabsf(x.y)), splat2(kRsqrt2));
  const float2 q = fma2(splat2(0.5f), w, splat2(1.0f));
  const float2 t = make_float2(rcp_approx(q.x), rcp_approx(q.y));
  const float2 p = erfc_poly(t);
  const float2 e = mul2(fma2(make_float2(-w.x, -w.y), w, p), splat2(kLog2e));
  const float2 h = mul2(mul2(splat2(0.5f), t), make_float2(Elem<T>::exp2(e.x), Elem<T>::exp2(e.y)));
  const float2 om = add2(splat2(1.0f), make_float2(-h.x, -h.y));  // 1 - h
  float2 y = mul2(x, make_float2(x.x >= 0.0f ? om.x : h.x, x.y >= 0.0f ? om.y : h.y));
  y.x = (x.x == -INFINITY) ? -0.0f : y.x;
  y.y = (x.y == -INFINITY) ? -0.0f : y.y;
  return y;
}

template <typename T, int KIND>
__device__ __forceinline__ float2 gelu_f2(float2 x) {
  return KIND == FK_GELU_TANH ? gelu_tanh_f2<T>(x) : gelu_erf_f2<T>(x);
}

template <typename T, int KIND>
__device__ __forceinline__ float gelu_f(float x) {
  return KIND == FK_GELU_TANH ? gelu_tanh_f<T>(x) : gelu_erf_f<T>(x);
}

}  // namespace
}  // namespace fk
