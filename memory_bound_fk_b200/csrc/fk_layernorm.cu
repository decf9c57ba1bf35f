// fk_layernorm.cu -- LayerNorm over rows, with an optional affine step and
// an optional GELU epilogue, fused into one pass over HBM (sm_100a).
//
// What is computed: the normalisation step of the fused LayerNorm -> Linear
// -> GELU example of lecture 6, "GPU Kernels and Triton" (cs336.sjfarmltd.com),
// sections 6.1-6.2 (F.layer_norm over the last axis): for each row of a
// row-major [rows, cols] matrix,
//     mean = sum_j x_j / cols,  var = sum_j (x_j - mean)^2 / cols,
//     y_j  = (x_j - mean) / sqrt(var + eps) * gamma_j + beta_j,
// then GELU(y_j) when asked.  Unfused, the three steps cost three reads and
// three writes of the activations (section 6.1); here the row is read once
// and written once.
//
// The row sits in registers as its packed 16-byte words (the row I/O of
// fk_rows.cuh), widened to fp32 as each pass uses it, and is reduced twice
// without touching HBM again:
//   pass 1: m1 = sum_j x_j / cols (a first, fp32-rounded estimate);
//   pass 2: a = sum_j (x_j - m1), b = sum_j (x_j - m1)^2, one paired reduction;
//           d = a / cols corrects m1 (mean = m1 + d) and
//           var = b / cols - d^2 (d is only m1's rounding error, so nothing
//           cancels);
//   output: y_j = (x_j - m1) rstd - d rstd, rstd = rsqrt(var + eps) (one
//           FMA; d rstd, a tiny term, is rounded once per row), affine, GELU.
// x_j - m1 is exact to a rounding relative to itself, so the error of y does
// not grow with |mean| / std the way a single fp32 mean's rounding would
// make it.
//
// Three shapes, chosen by row length as for softmax: one warp per row (up to
// 1024 columns; a forced warp plan holds up to 1024 fp32 / 2048 bf16), one
// block per row (up to 32768 columns),
// and for longer rows one 512-thread block per row that streams the row
// twice: a statistics pass that keeps a running (count, mean, M2) of x - p
// per thread (p: the mean of the row's first chunk), merging each
// 16-element chunk's exact two-pass statistics with the pairwise rule of
// Chan, Golub and LeVeque (1979), then a normalising pass.
#include <cuda_bf16.h>

#include "fk_common.cuh"
#include "fk_gelu.cuh"
#include "fk_internal.h"
#include "fk_rows.cuh"

namespace fk {
namespace {

constexpr int kLnStreamThreads = 512;
constexpr int kLnStreamElems = 16;  // elements per thread per streamed chunk
constexpr size_t kLnMaxGrid = 0x7fffffffu;

// Is element k of chunk c of thread t a column of the row?  (The placement
// of load_chunks: aligned rows hold whole vectors -- cols is a multiple of
// VEC there -- so the vector index decides; the scalar path interleaves by
// TEAM.)
template <typename T, int TEAM, bool ALIGNED, typename Idx>
__device__ __forceinline__ bool col_of(Idx vfirst, int c, int k, int t, Idx cols, Idx* col) {
  constexpr int VEC = Elem<T>::VEC;
  Idx e;
  if constexpr (ALIGNED) {
    e = (vfirst + static_cast<Idx>(c) * TEAM + t) * VEC + k;
  } else {
    e = (vfirst + static_cast<Idx>(c) * TEAM) * VEC + t + static_cast<Idx>(k) * TEAM;
  }
  *col = e;
  return e < cols;
}

// The same test with one comparison per vector on the aligned path.
template <typename T, int TEAM, bool ALIGNED, typename Idx>
__device__ __forceinline__ bool in_row(Idx vfirst, int c, int k, int t, Idx cols) {
  constexpr int VEC = Elem<T>::VEC;
  if constexpr (ALIGNED) {
    (void)k;
    return (vfirst + static_cast<Idx>(c) * TEAM + t) * VEC < cols;
  } else {
    Idx col;
    return col_of<T, TEAM, false>(vfirst, c, k, t, cols, &col);
  }
}

// Value k of a packed 16-byte word (4 fp32 or 8 bf16 values).  Rows stay
// packed in registers and are widened as each pass uses them: for bf16 this
// halves the registers a row takes, so more rows are in flight per SM.  The
// widening is a volatile asm so that the compiler redoes it in every pass
// (one instruction) instead of keeping all widened values live.
template <typename T>
__device__ __forceinline__ float val(const uint4& w, int k) {
  if constexpr (sizeof(T) == 4) {
    const uint32_t u = k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w;
    return __uint_as_float(u);
  } else {
    const uint32_t u = k < 2 ? w.x : k < 4 ? w.y : k < 6 ? w.z : w.w;
    uint32_t r;
    if (k & 1) {
      asm volatile("and.b32 %0, %1, 0xffff0000;" : "=r"(r) : "r"(u));
    } else {
      asm volatile("shl.b32 %0, %1, 16;" : "=r"(r) : "r"(u));
    }
    return __uint_as_float(r);
  }
}

// (x_k + c, x_k+1 + c) for the pair of values k, k + 1 (k even) of a packed
// word, each rounded once to fp32.  bf16: two sm_100 mixed-precision adds
// (add.f32.bf16 takes the bf16 half of the word as it is), one instruction
// per value where widening first took two per pair more.  The results are
// those of widening (exact) and adding.
template <typename T>
__device__ __forceinline__ float2 add_pair(const uint4& w, int k, float2 c) {
  if constexpr (sizeof(T) == 4) {
    return add2(make_float2(val<T>(w, k), val<T>(w, k + 1)), c);
  } else {
    const uint32_t u = k < 2 ? w.x : k < 4 ? w.y : k < 6 ? w.z : w.w;
    float2 d;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %3;\n\tadd.rn.f32.bf16 %1, hi, %4;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "r"(u), "f"(c.x), "f"(c.y));
    return d;
  }
}

// 16-byte read-only load that stays in program order with the row's
// (volatile) stores, so the compiler fetches each chunk's parameters just
// before that chunk is stored instead of hoisting every chunk's parameters
// into registers at once.
__device__ __forceinline__ float4 ld_param_v4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

// gamma / beta of the VEC columns of chunk c of thread t, fp32 (nullptr:
// the default).  On the aligned path a vector's parameters are VEC / 4
// float4 loads; they are the same for every row, so they come from L1 / L2,
// not HBM.
template <typename T, int TEAM, bool ALIGNED, typename Idx>
__device__ __forceinline__ void load_affine(const float* p, float dflt, Idx vfirst, int c, Idx cols, int t,
                                            float* out) {
  constexpr int VEC = Elem<T>::VEC;
  if (p == nullptr) {
#pragma unroll
    for (int k = 0; k < VEC; ++k) out[k] = dflt;
    return;
  }
  if constexpr (ALIGNED) {
    const Idx e0 = (vfirst + static_cast<Idx>(c) * TEAM + t) * VEC;
#pragma unroll
    for (int q = 0; q < VEC / 4; ++q) {
      float4 g = make_float4(dflt, dflt, dflt, dflt);
      if (e0 < cols) g = ld_param_v4(p + e0 + 4 * q);
      out[4 * q + 0] = g.x;
      out[4 * q + 1] = g.y;
      out[4 * q + 2] = g.z;
      out[4 * q + 3] = g.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      Idx col;
      out[k] = col_of<T, TEAM, false>(vfirst, c, k, t, cols, &col) ? __ldg(p + col) : dflt;
    }
  }
}

// The epilogue, on a pair of values.  GELU takes the flush-to-zero
// exponential for either output type: a GELU output below 2^-126 is within
// the LayerNorm error bound of 0.
template <int EPI>
__device__ __forceinline__ float2 epilogue2(float2 z) {
  if constexpr (EPI == FK_EPILOGUE_GELU_TANH) {
    return gelu_tanh_f2<float>(z);
  } else if constexpr (EPI == FK_EPILOGUE_GELU_ERF) {
    return gelu_erf_f2<float>(z);
  } else {
    return z;
  }
}

// y = ((x - m1) rstd - d rstd) * gamma + beta, then the epilogue, stored
// chunk by chunk (only one chunk's gamma / beta are live at a time).
template <typename T, int VPT, int TEAM, bool ALIGNED, int EPI, typename Idx>
__device__ __forceinline__ void normalise_store(T* yr, const uint4* raw, float m1, float d, float rstd,
                                                const float* gamma, const float* beta, Idx vfirst, Idx ve,
                                                Idx cols, int t) {
  constexpr int VEC = Elem<T>::VEC;
  const float ndr = -d * rstd;
  store_chunks_fn<T, VPT, TEAM, ALIGNED, Idx>(yr, vfirst, ve, cols, t, [&](int c, float* o) {
    float g[VEC], b[VEC];
    load_affine<T, TEAM, ALIGNED, Idx>(gamma, 1.0f, vfirst, c, cols, t, g);
    load_affine<T, TEAM, ALIGNED, Idx>(beta, 0.0f, vfirst, c, cols, t, b);
    // pairs of columns, each lane as ((x - m1) rstd - d rstd) * gamma + beta
#pragma unroll
    for (int k = 0; k < VEC; k += 2) {
      float2 z = add_pair<T>(raw[c], k, splat2(-m1));
      z = fma2(z, splat2(rstd), splat2(ndr));
      z = epilogue2<EPI>(fma2(z, make_float2(g[k], g[k + 1]), make_float2(b[k], b[k + 1])));
      o[k] = z.x;
      o[k + 1] = z.y;
    }
  });
}

// Sum of the values a thread holds (padding is +0).
template <typename T, int VPT>
__device__ __forceinline__ float sum_raw(const uint4* raw) {
  constexpr int VEC = Elem<T>::VEC;
  // four accumulators (column k into k % 4), two per packed pair
  float2 s01 = make_float2(0.0f, 0.0f), s23 = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int c = 0; c < VPT; ++c)
#pragma unroll
    for (int k = 0; k < VEC; k += 2) {
      if (k & 2)
        s23 = add_pair<T>(raw[c], k, s23);
      else
        s01 = add_pair<T>(raw[c], k, s01);
    }
  return (s01.x + s01.y) + (s23.x + s23.y);
}

// Pass-2 partial sums of one thread: sum (x - m1) and sum (x - m1)^2 over
// its columns of the row (padding excluded).  FULL: every value the thread
// holds is a column of the row (no padding to mask).
template <typename T, int VPT, int TEAM, bool ALIGNED, typename Idx, bool FULL = false>
__device__ __forceinline__ float2 centred_sums(const uint4* raw, float m1, Idx vfirst, Idx cols, int t) {
  constexpr int VEC = Elem<T>::VEC;
  // two accumulators each (even and odd columns), one packed pair
  float2 a = make_float2(0.0f, 0.0f), b = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
#pragma unroll
    for (int k = 0; k < VEC; k += 2) {
      float2 z = add_pair<T>(raw[c], k, splat2(-m1));
      if (!FULL) {
        z.x = in_row<T, TEAM, ALIGNED>(vfirst, c, k, t, cols) ? z.x : 0.0f;
        z.y = in_row<T, TEAM, ALIGNED>(vfirst, c, k + 1, t, cols) ? z.y : 0.0f;
      }
      a = add2(a, z);
      b = fma2(z, z, b);
    }
  }
  return make_float2(a.x + a.y, b.x + b.y);
}

// ---------------------------------------------------------------- warp path

template <typename T, int VPT, bool ALIGNED, int EPI>
__global__ void __launch_bounds__(kWarpThreads)
    layernorm_warp_kernel(const T* x, T* y, const float* gamma, const float* beta, size_t rows, int cols,
                          float eps) {
  constexpr int VEC = Elem<T>::VEC;
  const int lane = threadIdx.x & 31;
  const int nvec = (cols + VEC - 1) / VEC;
  const float inv_n = 1.0f / static_cast<float>(cols);
  const unsigned rpb = blockDim.x >> 5;  // rows (= warps) per block
  const size_t stride = static_cast<size_t>(gridDim.x) * rpb;
  for (size_t row = static_cast<size_t>(blockIdx.x) * rpb + (threadIdx.x >> 5); row < rows; row += stride) {
    const T* xr = x + row * static_cast<size_t>(cols);
    T* yr = y + row * static_cast<size_t>(cols);
    uint4 raw[VPT];
    load_chunks<T, VPT, 32, ALIGNED, false, int, true>(xr, 0, nvec, cols, cols, lane, raw);
    const float m1 = warp_sum(sum_raw<T, VPT>(raw)) * inv_n;
    float2 ab = centred_sums<T, VPT, 32, ALIGNED, int>(raw, m1, 0, cols, lane);
    ab.x = warp_sum(ab.x);
    ab.y = warp_sum(ab.y);
    const float d = ab.x * inv_n;
    const float rstd = rsqrtf(fmaxf(fmaf(-d, d, ab.y * inv_n), 0.0f) + eps);
    normalise_store<T, VPT, 32, ALIGNED, EPI, int>(yr, raw, m1, d, rstd, gamma, beta, 0, nvec, cols, lane);
  }
}

// ---------------------------------------------------------------- block path

// Rows in flight per SM for 128-thread blocks, bought with registers:
// bf16 rows fit 64 registers without spills, eight blocks instead of
// seven; fp32 rows take 96 registers by default (five blocks).  Measured on
// B200 (16384 x 4096 fp32, gamma / beta, L2 cleaned): without an epilogue
// six blocks (80 registers, no spills) 89.2 us against 90.6 at five and
// 91.7 at seven; with the tanh GELU seven blocks (72 registers, a few
// spilled words) 88.7 against 90.1 at six and 102.5 at five; with the exact
// GELU 96.2 at seven, 102.1 at six, 108.5 at five.
template <typename T, int THREADS, int EPI>
constexpr int ln_block_min_blocks() {
  if (THREADS != 128) return 1;
  if (sizeof(T) == 2) return 8;
  return EPI == FK_EPILOGUE_NONE ? 6 : 7;
}

template <typename T, int THREADS, int EPT, bool ALIGNED, int EPI>
__global__ void __launch_bounds__(THREADS, ln_block_min_blocks<T, THREADS, EPI>())
    layernorm_block_kernel(const T* x, T* y, const float* gamma, const float* beta, size_t rows, int cols,
                           float eps) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = EPT / VEC;
  constexpr int NW = THREADS / 32;
  static_assert(VPT * VEC == EPT, "EPT must be a multiple of the vector width");
  __shared__ float red1[NW];
  __shared__ float2 red2[NW];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nvec = (cols + VEC - 1) / VEC;
  const float inv_n = 1.0f / static_cast<float>(cols);
  for (size_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const T* xr = x + row * static_cast<size_t>(cols);
    T* yr = y + row * static_cast<size_t>(cols);
    uint4 raw[VPT];
    load_chunks<T, VPT, THREADS, ALIGNED, false, int, true>(xr, 0, nvec, cols, cols, t, raw);
    float s = warp_sum(sum_raw<T, VPT>(raw));
    if (lane == 0) red1[warp] = s;
    __syncthreads();
    s = red1[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) s += red1[w];
    const float m1 = s * inv_n;

    // bf16 rows that fill every thread's vectors exactly need no padding
    // masks (issue-bound rows; fp32 rows keep one code path)
    float2 ab = (sizeof(T) == 2 && ALIGNED && nvec == VPT * THREADS)
                    ? centred_sums<T, VPT, THREADS, ALIGNED, int, true>(raw, m1, 0, cols, t)
                    : centred_sums<T, VPT, THREADS, ALIGNED, int>(raw, m1, 0, cols, t);
    ab.x = warp_sum(ab.x);
    ab.y = warp_sum(ab.y);
    if (lane == 0) red2[warp] = ab;
    __syncthreads();
    ab = red2[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      ab.x += red2[w].x;
      ab.y += red2[w].y;
    }
    const float d = ab.x * inv_n;
    const float rstd = rsqrtf(fmaxf(fmaf(-d, d, ab.y * inv_n), 0.0f) + eps);
    normalise_store<T, VPT, THREADS, ALIGNED, EPI, int>(yr, raw, m1, d, rstd, gamma, beta, 0, nvec, cols, t);
    __syncthreads();  // red1 / red2 are rewritten by the next row
  }
}

// ---------------------------------------------------------------- streaming path

// Running statistics of a set of values: count, mean, sum of squared
// deviations from the mean.
struct Moments {
  float n, mean, m2;
};

// Pairwise merge (Chan, Golub and LeVeque): the deviation of the two means
// enters M2 weighted by na * nb / n.
__device__ __forceinline__ Moments merge_moments(Moments a, Moments b) {
  const float n = a.n + b.n;
  if (n == 0.0f) return a;
  const float delta = b.mean - a.mean;
  const float wb = b.n / n;
  Moments r;
  r.n = n;
  r.mean = fmaf(delta, wb, a.mean);
  r.m2 = a.m2 + b.m2 + delta * delta * a.n * wb;
  return r;
}

template <int THREADS>
__device__ __forceinline__ Moments block_merge_moments(Moments m, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Moments q;
    q.n = __shfl_xor_sync(0xffffffffu, m.n, o);
    q.mean = __shfl_xor_sync(0xffffffffu, m.mean, o);
    q.m2 = __shfl_xor_sync(0xffffffffu, m.m2, o);
    m = merge_moments(m, q);
  }
  if (lane == 0) {
    red[3 * warp + 0] = m.n;
    red[3 * warp + 1] = m.mean;
    red[3 * warp + 2] = m.m2;
  }
  __syncthreads();
  Moments r = {red[0], red[1], red[2]};
#pragma unroll
  for (int w = 1; w < THREADS / 32; ++w) r = merge_moments(r, Moments{red[3 * w], red[3 * w + 1], red[3 * w + 2]});
  return r;
}

template <typename T, bool ALIGNED, int EPI>
__global__ void __launch_bounds__(kLnStreamThreads)
    layernorm_stream_kernel(const T* x, T* y, const float* gamma, const float* beta, size_t rows, size_t cols,
                            float eps) {
  constexpr int THREADS = kLnStreamThreads;
  constexpr int NW = THREADS / 32;
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = kLnStreamElems / VEC;
  constexpr size_t STEP = static_cast<size_t>(THREADS) * VPT;
  __shared__ float red[3 * NW];
  __shared__ float2 piv[NW];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t nvec = (cols + VEC - 1) / VEC;
  for (size_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const T* xr = x + row * cols;
    T* yr = y + row * cols;
    uint4 raw[VPT];
    // pivot p: the mean of the row's first chunk.  The moments below are
    // those of x - p, whose mean is of the order of the row's spread, so
    // its fp32 rounding is small against the spread even when |mean| is not.
    load_chunks<T, VPT, THREADS, ALIGNED, false, size_t, true>(xr, 0, nvec, cols, cols, t, raw);
    float cnt = 0.0f;
#pragma unroll
    for (int c = 0; c < VPT; ++c)
#pragma unroll
      for (int k = 0; k < VEC; ++k) {
        size_t col;
        cnt += col_of<T, THREADS, ALIGNED>(size_t{0}, c, k, t, cols, &col) ? 1.0f : 0.0f;
      }
    float2 sc = make_float2(warp_sum(sum_raw<T, VPT>(raw)), warp_sum(cnt));
    if (lane == 0) piv[warp] = sc;
    __syncthreads();
    sc = piv[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      sc.x += piv[w].x;
      sc.y += piv[w].y;
    }
    const float p = sc.x / sc.y;

    // pass 1: each chunk's exact two-pass moments of x - p, merged into a
    // running total (the first chunk is read again, from L2)
    Moments run = {0.0f, 0.0f, 0.0f};
    for (size_t c0 = 0; c0 < nvec; c0 += STEP) {
      load_chunks<T, VPT, THREADS, ALIGNED, false, size_t, true>(xr, c0, nvec, cols, cols, t, raw);
      float n = 0.0f, s = 0.0f;
#pragma unroll
      for (int c = 0; c < VPT; ++c)
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
          size_t col;
          const bool in = col_of<T, THREADS, ALIGNED>(c0, c, k, t, cols, &col);
          n += in ? 1.0f : 0.0f;
          s += in ? val<T>(raw[c], k) - p : 0.0f;
        }
      if (n > 0.0f) {
        // centre the chunk on cc ~ its mean; ab.x / n is what cc misses by,
        // and (cc - p) is exact when cc and p are within a factor of two
        const float cc = p + s / n;
        const float2 ab = centred_sums<T, VPT, THREADS, ALIGNED, size_t>(raw, cc, c0, cols, t);
        const float dc = ab.x / n;
        run = merge_moments(run, Moments{n, (cc - p) + dc, fmaxf(fmaf(-dc, ab.x, ab.y), 0.0f)});
      }
    }
    const Moments tot = block_merge_moments<THREADS>(run, red);
    const float rstd = rsqrtf(tot.m2 / tot.n + eps);
    // pass 2: normalise ((x - p) - mean of (x - p)) and store
    for (size_t c0 = 0; c0 < nvec; c0 += STEP) {
      load_chunks<T, VPT, THREADS, ALIGNED, false, size_t, true>(xr, c0, nvec, cols, cols, t, raw);
      normalise_store<T, VPT, THREADS, ALIGNED, EPI, size_t>(yr, raw, p, tot.mean, rstd, gamma, beta, c0, nvec,
                                                             cols, t);
    }
    __syncthreads();  // red and piv are rewritten by the next row
  }
}

// ---------------------------------------------------------------- launchers

struct LnArgs {
  const void* x;
  void* y;
  const float* gamma;
  const float* beta;
  size_t rows, cols;
  float eps;
};

template <typename T, bool ALIGNED, int EPI>
cudaError_t launch_ln_warp(const LnArgs& a, int threads, int vpt, cudaStream_t s) {
  const size_t rpb = static_cast<size_t>(threads) / 32;
  size_t blocks = (a.rows + rpb - 1) / rpb;
  if (blocks > kLnMaxGrid) blocks = kLnMaxGrid;
  const T* x = static_cast<const T*>(a.x);
  T* y = static_cast<T*>(a.y);
  const int c = static_cast<int>(a.cols);
  const unsigned g = static_cast<unsigned>(blocks);
  switch (vpt) {
    case 1: layernorm_warp_kernel<T, 1, ALIGNED, EPI><<<g, threads, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    case 2: layernorm_warp_kernel<T, 2, ALIGNED, EPI><<<g, threads, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    case 4: layernorm_warp_kernel<T, 4, ALIGNED, EPI><<<g, threads, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    case 8: layernorm_warp_kernel<T, 8, ALIGNED, EPI><<<g, threads, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T, int EPT, bool ALIGNED, int EPI>
cudaError_t launch_ln_block_ept(const LnArgs& a, int threads, cudaStream_t s) {
  const unsigned g = static_cast<unsigned>(a.rows < kLnMaxGrid ? a.rows : kLnMaxGrid);
  const T* x = static_cast<const T*>(a.x);
  T* y = static_cast<T*>(a.y);
  const int c = static_cast<int>(a.cols);
  switch (threads) {
    case 128: layernorm_block_kernel<T, 128, EPT, ALIGNED, EPI><<<g, 128, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    case 256: layernorm_block_kernel<T, 256, EPT, ALIGNED, EPI><<<g, 256, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    case 512: layernorm_block_kernel<T, 512, EPT, ALIGNED, EPI><<<g, 512, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    case 1024: layernorm_block_kernel<T, 1024, EPT, ALIGNED, EPI><<<g, 1024, 0, s>>>(x, y, a.gamma, a.beta, a.rows, c, a.eps); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T, bool ALIGNED, int EPI>
cudaError_t launch_ln_plan(const LnArgs& a, const fk_softmax_plan& p, cudaStream_t s) {
  switch (p.path) {
    case FK_PATH_WARP: return launch_ln_warp<T, ALIGNED, EPI>(a, p.threads, p.vpt, s);
    case FK_PATH_CTA:
      switch (p.vpt * Elem<T>::VEC) {
        case 16: return launch_ln_block_ept<T, 16, ALIGNED, EPI>(a, p.threads, s);
        case 32: return launch_ln_block_ept<T, 32, ALIGNED, EPI>(a, p.threads, s);
        default: return cudaErrorInvalidValue;
      }
    case FK_PATH_TWOPHASE: {
      const unsigned g = static_cast<unsigned>(a.rows < kLnMaxGrid ? a.rows : kLnMaxGrid);
      layernorm_stream_kernel<T, ALIGNED, EPI><<<g, kLnStreamThreads, 0, s>>>(
          static_cast<const T*>(a.x), static_cast<T*>(a.y), a.gamma, a.beta, a.rows, a.cols, a.eps);
      return cudaGetLastError();
    }
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, bool ALIGNED>
cudaError_t launch_ln_epi(const LnArgs& a, int epilogue, const fk_softmax_plan& p, cudaStream_t s) {
  switch (epilogue) {
    case FK_EPILOGUE_NONE: return launch_ln_plan<T, ALIGNED, FK_EPILOGUE_NONE>(a, p, s);
    case FK_EPILOGUE_GELU_TANH: return launch_ln_plan<T, ALIGNED, FK_EPILOGUE_GELU_TANH>(a, p, s);
    case FK_EPILOGUE_GELU_ERF: return launch_ln_plan<T, ALIGNED, FK_EPILOGUE_GELU_ERF>(a, p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_layernorm(const void* x, void* y, const float* gamma, const float* beta, size_t rows,
                             size_t cols, int dtype, float eps, int epilogue, const fk_softmax_plan& plan,
                             bool aligned, cudaStream_t stream) {
  const LnArgs a = {x, y, gamma, beta, rows, cols, eps};
  if (dtype == FK_F32) {
    return aligned ? launch_ln_epi<float, true>(a, epilogue, plan, stream)
                   : launch_ln_epi<float, false>(a, epilogue, plan, stream);
  }
  return aligned ? launch_ln_epi<__nv_bfloat16, true>(a, epilogue, plan, stream)
                 : launch_ln_epi<__nv_bfloat16, false>(a, epilogue, plan, stream);
}

}  // namespace fk
