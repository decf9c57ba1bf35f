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

// Inputs below kGeluFloor are raised to it first, by a NaN-propagating max
// (one instruction): both forms give -0 from there down, the correctly
// rounded value (|GELU(x)| < 1e-49 for x <= -15, below every fp32 and bf16
// subnormal), and x = -inf no longer meets inf * 0 on the way.
constexpr float kGeluFloor = -30.0f;

__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// The same on a packed bf16 pair, to the floor of the form used for bf16
// outputs (both exact in bf16: -30 = 0xc1f0, -11 = 0xc130).
template <int KIND>
__device__ __forceinline__ uint32_t max_nan_floor_bf16x2(uint32_t w) {
  constexpr uint32_t kFloorPair = KIND == FK_GELU_TANH ? 0xc130c130u : 0xc1f0c1f0u;
  uint32_t r;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(kFloorPair));
  return r;
}

// 1/s on the FMA pipes, for s in [2^-125, 2^125]: an estimate from the bits,
// K - bits(s) with K = 0x7ef311c0 (the constant of smallest largest relative
// error over a scan of the mantissa, 5.1%), then two Newton steps
// r <- r + r (1 - s r), each squaring the relative error: under 1e-5, far
// below a bf16 half ulp (2^-9).  Four FMAs and an integer subtraction in
// place of one MUFU.RCP, for kernels that MUFU limits.
constexpr uint32_t kRecipMagic = 0x7ef311c0u;

__device__ __forceinline__ float recip_newton(float s) {
  float r = __uint_as_float(kRecipMagic - __float_as_uint(s));
  r = fmaf(r, fmaf(-s, r, 1.0f), r);
  return fmaf(r, fmaf(-s, r, 1.0f), r);
}

__device__ __forceinline__ float2 recip_newton2(float2 s) {
  const float2 ns = make_float2(-s.x, -s.y);
  float2 r = make_float2(__uint_as_float(kRecipMagic - __float_as_uint(s.x)),
                         __uint_as_float(kRecipMagic - __float_as_uint(s.y)));
  r = fma2(r, fma2(ns, r, splat2(1.0f)), r);
  return fma2(r, fma2(ns, r, splat2(1.0f)), r);
}

// Exponent offset of the GELU tails.  bf16 outputs keep values down to
// 2^-133, so their tail terms are taken 2^64 too large, where the
// flush-to-zero MUFU units (one instruction each; the forms that keep
// subnormal results take several) cannot flush them, and are scaled back by
// 2^-64 in one rounding before the last product.  Folding the offset into
// an exponent rounds it to 2^-18 absolute, a relative error under 2e-6 of
// the exponential: far below a bf16 ulp.  fp32 outputs take the terms
// flushed below 2^-126 (an absolute error under 1.2e-38 after the product).
//
// bf16 outputs of the tanh form take their reciprocal on the FMA pipes
// (recip_newton: the elementwise bf16 kernel is bound by MUFU, two
// operations per value), which wants a finite sum: inputs are raised to -11
// instead of -30 (2^(a - 64) <= 2^98 there; every x <= -10.4 gives -0
// already, the correctly rounded bf16 value).
template <typename T>
struct GeluScale {
  static constexpr float kBias = 0.0f;
  static constexpr float kUnbias = 1.0f;
  static constexpr float kTanhFloor = kGeluFloor;
  static constexpr bool kNewtonRecip = false;
};
template <>
struct GeluScale<__nv_bfloat16> {
  static constexpr float kBias = 64.0f;
  static constexpr float kUnbias = 0x1p-64f;
  static constexpr float kTanhFloor = -11.0f;
  static constexpr bool kNewtonRecip = true;
};

// tanh form: 0.5 x (1 + tanh u) = x sigma(2u) = x / (1 + 2^a) with
// a = -2u log2(e) (< 0 for x > 0).  For x < 0 the quotient is the small
// tail itself, without cancellation; where 2^a overflows it is 0 and y is
// -0, where 2^a flushes y is x.  One MUFU.EX2 and one MUFU.RCP.  With the
// offset the sum is 2^-64 + 2^(a-64), whose reciprocal 2^64 / (1 + 2^a)
// stays normal where 1 / (1 + 2^a) is subnormal (the flush-to-zero MUFU.RCP
// would drop it); 2^-64 is applied to that reciprocal, not to x q, which
// would overflow for x > 2^64.
template <typename T>
__device__ __forceinline__ float gelu_tanh_f(float x) {
  using S = GeluScale<T>;
  x = max_nan(x, S::kTanhFloor);
  const float p = fmaf(kB, x * x, kA);
  const float e = ex2_ftz(S::kBias != 0.0f ? fmaf(x, p, -S::kBias) : x * p);  // 2^(a - bias)
  const float sum = e + S::kUnbias;
  const float q = (S::kNewtonRecip ? recip_newton(sum) : rcp_approx(sum)) * S::kUnbias;  // 1 / (1 + 2^a)
  return x * q;
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
// where h is tiny (the fp32 rounding of the exponent, up to ~100).  bf16
// outputs use a degree-5 fit (below).
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

// The degree-5 fit (fit_erfc.py 5: largest error 6.0e-5, a relative error
// of erfc) for bf16 outputs, whose half ulp is 2^-9: over all 65536 bf16
// inputs it keeps every output within 1 ulp of the correctly rounded value
// (99.8% equal to it), four FMAs fewer than the fp32 fit.
template <typename V>
__device__ __forceinline__ V erfc_poly5(V t) {
  V p = splat_v<V>(1.878218204e-01f);
  p = fma_v(p, t, -5.907187462e-01f);
  p = fma_v(p, t, 3.472201824e-01f);
  p = fma_v(p, t, 3.165734410e-01f);
  p = fma_v(p, t, 1.004653573e+00f);
  p = fma_v(p, t, -1.265572071e+00f);
  return p;
}

template <typename T, typename V>
__device__ __forceinline__ V erfc_poly_for(V t) {
  if constexpr (sizeof(T) == 2)
    return erfc_poly5(t);
  else
    return erfc_poly(t);
}

// Phi(x) from the tail h: 1 - h for x >= 0, h for x < 0, as
// fma(s, h, (1 - s) / 2) with s = -1 or +1 taken from the sign bit of x
// (one logic instruction; -0 counts as negative, which gives the same -0
// output).  1 - h is rounded once, h is exact: the values of the select.
__device__ __forceinline__ float phi_sign(float x) {
  return __uint_as_float((__float_as_uint(x) & 0x80000000u) ^ 0xbf800000u);
}

template <typename T>
__device__ __forceinline__ float gelu_erf_f(float x) {
  using S = GeluScale<T>;
  x = max_nan(x, kGeluFloor);
  const float w = fabsf(x) * kRsqrt2;
  const float t = rcp_approx(fmaf(0.5f, w, 1.0f));
  const float p = erfc_poly_for<T>(t);
  const float hb = ex2_ftz(fmaf(fmaf(-w, w, p), kLog2e, S::kBias));  // 2^bias erfc(w) / t
  const float h = (0.5f * t * hb) * S::kUnbias;
  const float sg = phi_sign(x);
  return x * fmaf(sg, h, fmaf(sg, -0.5f, 0.5f));
}

// The two forms on a pair of values: every lane takes the operations of the
// scalar functions above in the same order (packed fp32 arithmetic rounds
// each lane as the scalar instruction does), so the results are identical,
// with about half the arithmetic instructions.
// CLAMPED: the caller has already raised x to kGeluFloor (bf16 inputs are
// clamped while still packed, one instruction per pair).
template <typename T, bool CLAMPED = false>
__device__ __forceinline__ float2 gelu_tanh_f2(float2 x) {
  using S = GeluScale<T>;
  if (!CLAMPED) x = make_float2(max_nan(x.x, S::kTanhFloor), max_nan(x.y, S::kTanhFloor));
  const float2 p = fma2(splat2(kB), mul2(x, x), splat2(kA));
  const float2 a = S::kBias != 0.0f ? fma2(x, p, splat2(-S::kBias)) : mul2(x, p);
  const float2 s = add2(make_float2(ex2_ftz(a.x), ex2_ftz(a.y)), splat2(S::kUnbias));
  float2 q;
  if constexpr (S::kNewtonRecip)
    q = recip_newton2(s);
  else
    q = make_float2(rcp_approx(s.x), rcp_approx(s.y));
  if constexpr (S::kBias != 0.0f) q = mul2(q, splat2(S::kUnbias));
  return mul2(x, q);
}

template <typename T, bool CLAMPED = false>
__device__ __forceinline__ float2 gelu_erf_f2(float2 x) {
  using S = GeluScale<T>;
  if (!CLAMPED) x = make_float2(max_nan(x.x, kGeluFloor), max_nan(x.y, kGeluFloor));
  const float2 w = mul2(make_float2(fabsf(x.x), fabsf(x.y)), splat2(kRsqrt2));
  const float2 q = fma2(splat2(0.5f), w, splat2(1.0f));
  const float2 t = make_float2(rcp_approx(q.x), rcp_approx(q.y));
  const float2 p = erfc_poly_for<T>(t);
  const float2 e = fma2(fma2(make_float2(-w.x, -w.y), w, p), splat2(kLog2e), splat2(S::kBias));
  float2 h = mul2(mul2(splat2(0.5f), t), make_float2(ex2_ftz(e.x), ex2_ftz(e.y)));
  if constexpr (S::kBias != 0.0f) h = mul2(h, splat2(S::kUnbias));
  const float2 sg = make_float2(phi_sign(x.x), phi_sign(x.y));
  return mul2(x, fma2(sg, h, fma2(sg, splat2(-0.5f), splat2(0.5f))));
}

template <typename T, int KIND, bool CLAMPED = false>
__device__ __forceinline__ float2 gelu_f2(float2 x) {
  return KIND == FK_GELU_TANH ? gelu_tanh_f2<T, CLAMPED>(x) : gelu_erf_f2<T, CLAMPED>(x);
}

template <typename T, int KIND>
__device__ __forceinline__ float gelu_f(float x) {
  return KIND == FK_GELU_TANH ? gelu_tanh_f<T>(x) : gelu_erf_f<T>(x);
}

}  // namespace
}  // namespace fk
