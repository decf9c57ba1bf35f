// fk_f32x2.cuh -- two fp32 values per instruction: the sm_100 packed
// add.rn / mul.rn / fma.rn .f32x2.  Each lane is rounded as the scalar
// operation would round it, so a pairwise rewrite of scalar code that keeps
// every lane's operations and their order gives bit-identical results with
// half the arithmetic instructions.
#pragma once

namespace fk {
namespace {

__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// Horner steps written once for one value or a pair.
__device__ __forceinline__ float fma_v(float p, float t, float c) { return fmaf(p, t, c); }
__device__ __forceinline__ float2 fma_v(float2 p, float2 t, float c) { return fma2(p, t, splat2(c)); }
template <typename V>
__device__ __forceinline__ V splat_v(float c);
template <>
__device__ __forceinline__ float splat_v<float>(float c) {
  return c;
}
template <>
__device__ __forceinline__ float2 splat_v<float2>(float c) {
  return splat2(c);
}

}  // namespace
}  // namespace fk
