// fk_common.cuh -- device helpers shared by the libfk kernels (sm_100a).
//
// Element traits for 16-byte vector I/O (fp32: 4 per vector, bf16: 8 per
// vector), streaming loads/stores, the base-2 exponential and the warp
// reductions.  Nothing here is used by, or uses, the CPU oracle.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace fk {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e), rounded to fp32

// ---------------------------------------------------------------- math

// 2^v with the MUFU.EX2 unit; subnormal results kept (no flush to zero).
__device__ __forceinline__ float ex2(float v) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// 2^v, subnormal results flushed to zero (where they cannot matter).
__device__ __forceinline__ float ex2_ftz(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// 1/v with MUFU.RCP, at most 1 ulp off; results below 2^-126 flush to
// zero and 1/inf is 0 (every softmax normaliser here is >= 1).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- I/O

// Read-only, do-not-keep-in-L1 128-bit load.  The memory clobber keeps the
// compiler from moving it across the stores of the same thread (in-place
// operation reads an element before it overwrites it).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// 128-bit store with the streaming (evict-first) cache hint.
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Predicated forms: the access happens only when `pred` holds (the address
// is not touched otherwise).  Keeping the predicate inside one asm statement,
// instead of branching around the access, lets the compiler interleave the
// stores with the arithmetic that produces them; with branches it hoists all
// of that arithmetic first and the register count of the row kernels nearly
// doubles.  A load that does not happen returns `fill` in every word.
__device__ __forceinline__ uint4 ld_stream_v4_if(const void* p, bool pred, uint32_t fill) {
  uint4 v = make_uint4(fill, fill, fill, fill);
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %5, 0;\n\t"
      "@q ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "l"(p), "r"(static_cast<unsigned>(pred))
      : "memory");
  return v;
}

__device__ __forceinline__ void st_stream_v4_if(void* p, uint4 v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %5, 0;\n\t"
      "@q st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};\n\t}" ::"l"(p),
      "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(static_cast<unsigned>(pred))
      : "memory");
}

// Max / sum of E register values with four independent accumulators, so the
// dependency chain is E/4 long instead of E.
template <int E>
__device__ __forceinline__ float max_of(const float* v) {
  float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int e = 0; e < E; ++e) a[e & 3] = fmaxf(a[e & 3], v[e]);
  return fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
}

template <typename T>
struct Elem;

// fp32: 4 values per 16-byte vector.
template <>
struct Elem<float> {
  static constexpr int VEC = 4;
  static constexpr uint32_t kNegInfWord = 0xff800000u;  // one -inf
  __device__ __forceinline__ static void unpack(uint4 v, float* o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 pack(const float* i) {
    return make_uint4(__float_as_uint(i[0]), __float_as_uint(i[1]), __float_as_uint(i[2]),
                      __float_as_uint(i[3]));
  }
  __device__ __forceinline__ static float load1(const float* p) { return __ldg(p); }
  __device__ __forceinline__ static void store1(float* p, float v) { *p = v; }
  // Keep the first `keep` values of a vector, -inf in the rest.
  __device__ __forceinline__ static uint4 keep_first(uint4 w, int keep) {
    w.x = keep > 0 ? w.x : kNegInfWord;
    w.y = keep > 1 ? w.y : kNegInfWord;
    w.z = keep > 2 ? w.z : kNegInfWord;
    w.w = keep > 3 ? w.w : kNegInfWord;
    return w;
  }
  // exp2 for softmax terms: results below 2^-126 flush to zero, an absolute
  // error under 1.2e-38 on an fp32 output (3% faster on 4096-column rows).
  __device__ __forceinline__ static float exp2(float a) { return ex2_ftz(a); }
  // Exponent offset of the single-reference (folded) path: none for fp32.
  static constexpr float kFoldBias = 0.0f;
  // 1 / (row sum), correctly rounded.  (MUFU.RCP alone made the compiler
  // schedule the 32-value rows into 76 registers or spills.)
  __device__ __forceinline__ static float recip(float s) { return __frcp_rn(s); }
  // Max of N raw vectors (4 independent accumulators).
  template <int N>
  __device__ __forceinline__ static float max_raw(const uint4* r) {
    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < N; ++i) {
      a[0] = fmaxf(a[0], __uint_as_float(r[i].x));
      a[1] = fmaxf(a[1], __uint_as_float(r[i].y));
      a[2] = fmaxf(a[2], __uint_as_float(r[i].z));
      a[3] = fmaxf(a[3], __uint_as_float(r[i].w));
    }
    return fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
  }
};

// bf16 (stored as raw 16-bit patterns): 8 values per 16-byte vector.
// Widening is exact (the pattern is the top half of an fp32); narrowing
// rounds to nearest even.
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int VEC = 8;
  static constexpr uint32_t kNegInfWord = 0xff80ff80u;  // two -inf
  __device__ __forceinline__ static void unpack2(uint32_t w, float* o) {
    o[0] = __uint_as_float(w << 16);
    o[1] = __uint_as_float(w & 0xffff0000u);
  }
  __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x -> low half
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static void unpack(uint4 v, float* o) {
    unpack2(v.x, o + 0);
    unpack2(v.y, o + 2);
    unpack2(v.z, o + 4);
    unpack2(v.w, o + 6);
  }
  __device__ __forceinline__ static uint4 pack(const float* i) {
    return make_uint4(pack2(i[0], i[1]), pack2(i[2], i[3]), pack2(i[4], i[5]), pack2(i[6], i[7]));
  }
  __device__ __forceinline__ static float load1(const __nv_bfloat16* p) {
    const unsigned short b = __ldg(reinterpret_cast<const unsigned short*>(p));
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
  __device__ __forceinline__ static void store1(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
  }
  // Keep the first `keep` values of a vector, -inf in the rest (word i holds
  // values 2i in its low half and 2i+1 in its high half).
  __device__ __forceinline__ static uint32_t keep_word(uint32_t w, int keep, int i) {
    return keep > 2 * i + 1 ? w : (keep > 2 * i ? ((w & 0xffffu) | 0xff800000u) : kNegInfWord);
  }
  __device__ __forceinline__ static uint4 keep_first(uint4 w, int keep) {
    return make_uint4(keep_word(w.x, keep, 0), keep_word(w.y, keep, 1), keep_word(w.z, keep, 2),
                      keep_word(w.w, keep, 3));
  }
  // exp2 for softmax terms: subnormal results kept, because bf16 outputs
  // down to 2^-133 must still round correctly.
  __device__ __forceinline__ static float exp2(float a) { return ex2(a); }
  // Single-reference (folded) path: exponentials are taken as 2^(a + 64)
  // with the flush-to-zero MUFU.EX2 (one instruction, against several for the
  // subnormal-preserving form).  The common factor 2^64 cancels against the
  // sum; terms whose unscaled value is below 2^-190 flush to 0, and their
  // correctly rounded bf16 output is 0 anyway (the smallest bf16 is 2^-133
  // and the normaliser is >= 1), while terms down to 2^-190 stay normal and
  // reach the bf16 subnormal range through the final multiplication.
  static constexpr float kFoldBias = 64.0f;
  // 1 / (row sum) with MUFU.RCP: at most 1 ulp off, invisible after rounding
  // to bf16; the sum is >= 2^64 here, so never subnormal.
  __device__ __forceinline__ static float recip(float s) { return rcp_approx(s); }
  // Max of N raw vectors with packed bf16x2 maximum (exact: the max of bf16
  // values is one of them).
  template <int N>
  __device__ __forceinline__ static float max_raw(const uint4* r) {
    __nv_bfloat162 a = __floats2bfloat162_rn(-INFINITY, -INFINITY), b = a;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162*>(&r[i].x));
      b = __hmax2(b, *reinterpret_cast<const __nv_bfloat162*>(&r[i].y));
      a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162*>(&r[i].z));
      b = __hmax2(b, *reinterpret_cast<const __nv_bfloat162*>(&r[i].w));
    }
    a = __hmax2(a, b);
    return fmaxf(__low2float(a), __high2float(a));
  }
};

}  // namespace fk
