// fk_softmax.cu -- row softmax kernels for sm_100a.
//
// What is computed (lecture 6, "GPU Kernels and Triton", cs336.sjfarmltd.com,
// section 7.2; CS336 lecture-6 notes, kyc001.github.io, section 5.2): for each
// row of a row-major [rows, cols] matrix, m = max_j x_j, l = sum_j exp(x_j - m),
// y_j = exp(x_j - m) / l.  exp(v) is evaluated as 2^(v log2 e) on MUFU.EX2 and
// the division as a multiplication by the correctly rounded 1/l.
//
// Four kernel shapes, chosen by row length (see fk_plan.cpp):
//   warp     -- one warp per row; the row sits in registers (up to 32 vectors
//               per lane-row, i.e. 1024 fp32 / 2048 bf16 columns);
//               max and sum by warp shuffles.
//   block    -- one thread block per row, 32 register-resident elements per
//               thread (up to 32768 columns); warp shuffles, then one shared
//               memory exchange between warps.
//   cluster  -- a thread-block cluster of 2..16 blocks per row, each block
//               holding a slice in registers (up to 64 values per thread);
//               each block reduces its slice to a partial (m_c, l_c), pushes
//               it into every other block's shared memory with st.async
//               (completing on the receiver's mbarrier), and merges the
//               partials with the running-max rule of section 7.2:
//               M = max_c m_c,  L = sum_c l_c exp(m_c - M).  Every element
//               is still read once and written once.  There is no cluster
//               barrier on the row path: the only one is split (arrive at
//               kernel start, wait just before the first push) and only
//               publishes the mbarrier initialisation.
//   twophase -- for rows longer than a cluster can hold: each block streams
//               its slice, keeping a per-thread running (m, l) (the online
//               recurrence of section 7.2), merges as above, then streams the
//               slice again to write exp(x - M) / L.  Three HBM transfers per
//               element instead of two.
//
// Placement within a row: a team of TEAM threads (a warp or a block) covers
// the row (or its slice) in chunks of TEAM 16-byte vectors.  On the vector
// path, thread t owns vector (chunk * TEAM + t), so a warp's loads are 512
// contiguous bytes.  When rows or pointers are not 16-byte aligned, the
// scalar path keeps the same chunks but gives thread t the elements
// chunk*TEAM*VEC + k*TEAM + t (k < VEC), which is again contiguous per warp.
//
// Special values: padding lanes hold -inf (exp gives 0, never stored);
// -inf inputs give exactly 0; a row that is all -inf gives 0/0 = NaN; a NaN
// is skipped by fmaxf but poisons the sum; a +inf gives inf - inf = NaN.
// Partial results of slices that are all -inf are merged without forming
// (-inf) - (-inf): see rescale().
//
// Scaled and causal form (every kernel, template flag SC): the exponent of
// x_j is scale * (x_j - m) and row r keeps only its first limit(r) columns
// (see row_limit); masked columns are never loaded -- their loads are
// predicated off, so they cost no HBM traffic -- and are written 0.  This is
// the score step of causal attention (lecture 6, "GPU Kernels and Triton",
// section 8: the scores times 1/sqrt(d_k), -inf where the key comes after
// the query, then the softmax) done in one pass, without an -inf tensor.
#include <cuda_bf16.h>

#include "fk_common.cuh"
#include "fk_internal.h"
#include "fk_rows.cuh"
#include "fk_sync.cuh"

namespace fk {

// Number of threads whose mbarrier wait gave up (see bounded_wait).
__device__ unsigned int g_wait_timeouts = 0;

namespace {

// Time limit of every mbarrier wait on the row paths.  A partner block that
// has not arrived after this long is not coming; the wait gives up, counts
// itself in g_wait_timeouts and the kernel finishes without hanging.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s

__device__ __noinline__ bool bounded_wait_slow(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > timeout_ns) {
      atomicAdd(&g_wait_timeouts, 1u);
      return false;
    }
  }
}

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity,
                                             uint64_t timeout_ns = kWaitTimeoutNs) {
  return mbar_try_wait(bar, parity) || bounded_wait_slow(bar, parity, timeout_ns);
}

// ---------------------------------------------------------------- merge rule

// exp(scale * (m_from - m_to)) for m_from <= m_to (k = scale * log2 e): the
// factor that moves a partial sum taken relative to max m_from onto max m_to.
// Equal maxima give exactly 1, which also covers (-inf, -inf) (an all -inf
// partial, whose sum is 0) and (+inf, +inf) (whose sum is already NaN).
__device__ __forceinline__ float rescale(float m_from, float m_to, float k) {
  return (m_from == m_to) ? 1.0f : ex2((m_from - m_to) * k);
}

// Reference point for exponentials of a partial whose max is m: m itself,
// or 0 for an all -inf partial (so that exp(-inf - ref) = 0, not NaN).
__device__ __forceinline__ float exp_ref(float m) { return (m == -INFINITY) ? 0.0f : m; }

// Columns kept in row `row` of the launch (see SoftmaxScaling): the query
// position of the row is (row0 + row) mod period + offset, and keys up to it
// are kept.  The host bounds period by the rows and offset by cols, so the
// sum cannot wrap.
// The 64-bit remainder, for periods or row indices of 2^32 and more, is a
// separate call: inlined, its instructions were issued for every row under a
// false predicate (a third of the extra instructions of causal 2048-column
// rows over plain ones, measured with ncu).
__device__ __noinline__ size_t row_limit_wide(size_t r, size_t period, size_t offset, size_t cols) {
  const size_t q = r % period + offset;
  return q < cols ? q + 1 : cols;
}

__device__ __forceinline__ size_t row_limit(const SoftmaxScaling& sc, size_t row, size_t cols) {
  if (sc.period == 0) return cols;
  if (!sc.fast32) return row_limit_wide(sc.row0 + row, sc.period, sc.offset, cols);
  const uint32_t n = static_cast<uint32_t>(sc.row0 + row);
  const uint32_t t = __umulhi(sc.magic, n);
  const uint32_t quot = (t + ((n - t) >> sc.shift1)) >> sc.shift2;
  const size_t q = static_cast<size_t>(n - quot * static_cast<uint32_t>(sc.period)) + sc.offset;
  return q < cols ? q + 1 : cols;
}

// row_limit for the kernels whose rows hold fewer than 2^31 columns, in
// 32-bit arithmetic (the offset is at most cols there, and fast32 means the
// period and every row index are below 2^32; the host leaves fast32 clear
// when there is no mask): one test and about ten integer instructions per
// row in the common case, where 64-bit arithmetic took about twice as many.
__device__ __forceinline__ int row_limit32(const SoftmaxScaling& sc, size_t row, int cols) {
  if (!sc.fast32) return static_cast<int>(row_limit(sc, row, static_cast<size_t>(cols)));
  const uint32_t n = static_cast<uint32_t>(sc.row0) + static_cast<uint32_t>(row);
  const uint32_t t = __umulhi(sc.magic, n);
  const uint32_t quot = (t + ((n - t) >> sc.shift1)) >> sc.shift2;
  const uint32_t rem = n - quot * static_cast<uint32_t>(sc.period);
  const uint32_t q = rem + static_cast<uint32_t>(sc.offset);  // wraps only when the sum exceeds cols anyway
  return (q >= rem && q < static_cast<uint32_t>(cols)) ? static_cast<int>(q) + 1 : cols;
}

// ---------------------------------------------------------------- row I/O

// Exponentials relative to ref, into v; returns their sum (four
// accumulators).  fp32 works in place on v (already unpacked at load); bf16
// unpacks the raw words as it goes, so the packed row is what stays live
// while the max is taken.
// FOLD (every exponential of the row shares the reference): one FMA and one
// flush-to-zero MUFU.EX2 per element, 2^(x log2 e - ref log2 e + bias); the
// rounding of ref*log2(e) and the 2^bias scale are common factors that
// cancel in the normalisation (bias: see Elem<T>::kFoldBias; the caller
// keeps |ref log2 e| below 2^24, see exp_sum_row).
// Otherwise (blocks or chunks with different references are merged later):
// (x - ref) is formed first, exact for the largest terms, and no bias is
// applied, so the partial sums of different references compare directly.
// k = scale * log2(e) (log2(e) for the plain softmax).  live: bit i clear
// when chunk i holds only masked columns (all -inf, see live_chunks); its
// terms are 0 and are not computed.
template <typename T, int VPT, bool FOLD>
__device__ __forceinline__ float exp_sum(const uint4* raw, float* v, float ref, float k, unsigned live = ~0u) {
  constexpr int VEC = Elem<T>::VEC;
  float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const float c = Elem<T>::kFoldBias - ref * k;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    if (((live >> i) & 1u) == 0u) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) v[i * VEC + j] = 0.0f;
      continue;
    }
    float f[VEC];
    if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) f[j] = v[i * VEC + j];
    } else {
      Elem<T>::unpack(raw[i], f);
    }
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const float e = FOLD ? ex2_ftz(fmaf(f[j], k, c)) : Elem<T>::exp2((f[j] - ref) * k);
      v[i * VEC + j] = e;
      s[j & 3] += e;
    }
  }
  return (s[0] + s[1]) + (s[2] + s[3]);
}

// Exponentials of values that all share the reference m, the max of the
// whole row.  The folded form takes 2^(x k - fl(m k)): the rounding error of
// fl(m k), up to |m k| 2^-24 in the exponent, scales every term of the row
// alike and cancels in the normalisation -- but only while it is small, or
// the terms overflow or flush.  So the row folds only when |m k| < 2^24 (an
// error of at most 1/2 in the exponent); rows with larger maxima (beyond
// about 1.2e7 at scale 1) take the unfolded form, one uniform branch per row.
template <typename T, int VPT>
__device__ __forceinline__ float exp_sum_row(const uint4* raw, float* v, float m, float k, unsigned live = ~0u) {
  if (fabsf(m * k) < 0x1p24f) return exp_sum<T, VPT, true>(raw, v, m, k, live);
  return exp_sum<T, VPT, false>(raw, v, exp_ref(m), k, live);
}

// Chunks of thread t that hold a column before lim (bit c for chunk c):
// under a causal mask the rest are wholly masked, so their exponentials
// need not be computed.  (Aligned rows: the thread's vector of the chunk;
// the scalar path: its first element.)
template <typename T, int VPT, int TEAM, bool ALIGNED, typename Idx>
__device__ __forceinline__ unsigned live_chunks(Idx vfirst, Idx lim, int t) {
  constexpr int VEC = Elem<T>::VEC;
  unsigned m = 0;
#pragma unroll
  for (int c = 0; c < VPT; ++c) {
    const Idx first = ALIGNED ? (vfirst + static_cast<Idx>(c) * TEAM + t) * VEC
                              : (vfirst + static_cast<Idx>(c) * TEAM) * VEC + t;
    m |= (first < lim ? 1u : 0u) << c;
  }
  return m;
}

// Max of the values a thread holds (after load_row).
template <typename T, int VPT>
__device__ __forceinline__ float row_max(const uint4* raw, const float* v) {
  if constexpr (sizeof(T) == 4) {
    return max_of<VPT * Elem<T>::VEC>(v);
  } else {
    return Elem<T>::template max_raw<VPT>(raw);
  }
}

// ---------------------------------------------------------------- warp path

template <typename T, int VPT, bool ALIGNED, bool SC>
__global__ void __launch_bounds__(kWarpThreads)
    softmax_warp_kernel(const T* x, T* y, size_t rows, int cols, SoftmaxScaling sc) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int E = VPT * VEC;
  const int lane = threadIdx.x & 31;
  const int nvec = (cols + VEC - 1) / VEC;
  const float k = SC ? sc.k : kLog2e;
  const unsigned rpb = blockDim.x >> 5;  // rows (= warps) per block
  const size_t stride = static_cast<size_t>(gridDim.x) * rpb;
  for (size_t row = static_cast<size_t>(blockIdx.x) * rpb + (threadIdx.x >> 5); row < rows; row += stride) {
    const T* xr = x + row * static_cast<size_t>(cols);
    T* yr = y + row * static_cast<size_t>(cols);
    uint4 raw[VPT];
    float v[E];
    const int lim = SC ? row_limit32(sc, row, cols) : cols;
    load_row<T, VPT, 32, ALIGNED, SC, int>(xr, 0, nvec, cols, lim, lane, raw, v);
    const float m = warp_max(row_max<T, VPT>(raw, v));
    const unsigned live = SC ? live_chunks<T, VPT, 32, ALIGNED, int>(0, lim, lane) : ~0u;
    const float s = warp_sum(exp_sum_row<T, VPT>(raw, v, m, k, live));
    store_chunks<T, VPT, 32, ALIGNED, int, SC>(yr, 0, nvec, cols, lane, v, Elem<T>::recip(s),
                                               sc.skip_masked ? lim : cols);
  }
}

// ---------------------------------------------------------------- cluster exchange

// Per-block partials of the row: inbox[i] receives block i's (max, sum);
// bar completes when the csize - 1 pushes from the other blocks have landed.
// Each cluster handles exactly one row, so every buffer is used once.
struct ClusterExchange {
  float2 inbox[kMaxCluster];
  uint64_t bar;
};

// Thread 0 of every block, before cluster_arrive_relaxed().
__device__ __forceinline__ void exchange_init(ClusterExchange& ex) {
  mbar_init(&ex.bar, 1);
  fence_mbarrier_init();
}

// All threads of the block, once per kernel.  Completes the start-up cluster
// barrier (so every receiver's mbarrier is initialised), pushes this
// block's (m, l) into every other block's inbox with st.async, waits
// (bounded) for the other blocks' pushes, and returns the merged (M, L) of
// the row.  When every partner arrives within the wait's limit, a block
// exits only after all pushes addressed to it have landed, and it pushes
// only to blocks that are waiting for it, so no block touches the shared
// memory of a block that has exited.  A wait that gives up (a partner did
// not arrive within 1 s) is counted in g_wait_timeouts and the block goes on
// with the partials it has; the call still returns FK_OK, so the count
// (fk_wait_timeouts) is how a caller learns that a row may be wrong.
__device__ __forceinline__ float2 exchange_merge(ClusterExchange& ex, float m, float l, int csize, int crank,
                                                 float k) {
  const int t = threadIdx.x, lane = t & 31;
  if (t == 0) mbar_arrive_expect_tx(&ex.bar, static_cast<uint32_t>(csize - 1) * 8u);
  cluster_wait();
  if (t < csize && t != crank) st_async_f2(cluster_addr(&ex.inbox[crank], t), m, l, cluster_addr(&ex.bar, t));
  bounded_wait(&ex.bar, 0);
  // every warp merges the partials itself: lane i takes block i's
  float mi = -INFINITY, li = 0.0f;
  if (lane < csize) {
    const float2 q = (lane == crank) ? make_float2(m, l) : ex.inbox[lane];
    mi = q.x;
    li = q.y;
  }
  const float M = warp_max(mi);
  const float L = warp_sum(lane < csize ? li * rescale(mi, M, k) : 0.0f);
  return make_float2(M, L);
}

// ---------------------------------------------------------------- block path

// One block per row; EPT = register-resident elements per thread.  Rows of
// 32 bytes per thread (16 bf16 values) keep few loads in flight per thread,
// so those kernels (up to 256 threads) are held to 2048 resident threads per
// SM (32 registers).
template <typename T, int THREADS, int EPT, bool ALIGNED, bool SC>
__global__ void __launch_bounds__(THREADS, (EPT * sizeof(T) <= 32 && THREADS <= 256 ? 2048 / THREADS : 1))
    softmax_block_kernel(const T* x, T* y, size_t rows, int cols, SoftmaxScaling sc) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = EPT / VEC;
  constexpr int E = VPT * VEC;
  constexpr int NW = THREADS / 32;
  static_assert(VPT * VEC == EPT, "EPT must be a multiple of the vector width");
  __shared__ float red_max[NW];
  __shared__ float red_sum[NW];

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nvec = (cols + VEC - 1) / VEC;
  const float k = SC ? sc.k : kLog2e;
  for (size_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const T* xr = x + row * static_cast<size_t>(cols);
    T* yr = y + row * static_cast<size_t>(cols);
    uint4 raw[VPT];
    float v[E];
    const int lim = SC ? row_limit32(sc, row, cols) : cols;
    load_row<T, VPT, THREADS, ALIGNED, SC, int>(xr, 0, nvec, cols, lim, t, raw, v);

    float m = warp_max(row_max<T, VPT>(raw, v));
    if (lane == 0) red_max[warp] = m;
    __syncthreads();
    m = red_max[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) m = fmaxf(m, red_max[w]);

    const unsigned live = SC ? live_chunks<T, VPT, THREADS, ALIGNED, int>(0, lim, t) : ~0u;
    float s = warp_sum(exp_sum_row<T, VPT>(raw, v, m, k, live));
    if (lane == 0) red_sum[warp] = s;
    __syncthreads();
    s = red_sum[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) s += red_sum[w];

    store_chunks<T, VPT, THREADS, ALIGNED, int, SC>(yr, 0, nvec, cols, t, v, Elem<T>::recip(s),
                                                    sc.skip_masked ? lim : cols);
    __syncthreads();  // red_max / red_sum are rewritten by the next row
  }
}

// ---------------------------------------------------------------- cluster path

// A cluster of csize blocks per row; block `rank` holds vectors
// [rank*per, (rank+1)*per) of the row in registers, per = ceil(nvec / csize).
// With 64 values a thread the plain aligned kernel's register budget is held
// so that more clusters are resident, and others stream while one waits at
// its exchange: fp32 to six 128-thread blocks an SM (three of 256; 80 vs 95
// registers, no spills; 512 x 131072 fp32 runs 80 instead of 86 us, and 7%
// slower again at seven), bf16 to eight (four of 256; 64 registers, no
// spills; 4096 x 65536 bf16 204 -> 191 us, 1024 x 131072 119 -> 107).  The
// scaled and the unaligned forms would spill under that bound and keep the
// default.
template <typename T, int THREADS, int EPT, bool PLAIN>
constexpr int cluster_min_blocks() {
  return PLAIN && EPT == 64 && THREADS <= 256 ? (sizeof(T) == 2 ? 1024 : 768) / THREADS : 1;
}

template <typename T, int THREADS, int EPT, bool ALIGNED, bool SC>
__global__ void __launch_bounds__(THREADS, cluster_min_blocks<T, THREADS, EPT, ALIGNED && !SC>())
    softmax_cluster_kernel(const T* x, T* y, size_t rows, int cols, SoftmaxScaling sc) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = EPT / VEC;
  constexpr int E = VPT * VEC;
  constexpr int NW = THREADS / 32;
  static_assert(VPT * VEC == EPT, "EPT must be a multiple of the vector width");
  __shared__ float red_max[NW];
  __shared__ float red_sum[NW];
  __shared__ __align__(16) ClusterExchange ex;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int csize = static_cast<int>(cluster_nctarank());
  const int crank = static_cast<int>(cluster_ctarank());
  const int nvec = (cols + VEC - 1) / VEC;
  const int per = (nvec + csize - 1) / csize;
  const int vb = imin(nvec, crank * per);
  const int ve = imin(nvec, vb + per);

  // one row per cluster (the host splits launches that would exceed the grid)
  const size_t row = blockIdx.x / csize;
  if (row >= rows) return;  // same for every block of the cluster
  if (t == 0) exchange_init(ex);
  cluster_arrive_relaxed();

  const T* xr = x + row * static_cast<size_t>(cols);
  T* yr = y + row * static_cast<size_t>(cols);
  const float k = SC ? sc.k : kLog2e;
  const int lim = SC ? row_limit32(sc, row, cols) : cols;
  uint4 raw[VPT];
  float v[E];
  load_row<T, VPT, THREADS, ALIGNED, SC, int>(xr, vb, ve, cols, lim, t, raw, v);

  float m = warp_max(row_max<T, VPT>(raw, v));
  if (lane == 0) red_max[warp] = m;
  __syncthreads();
  m = red_max[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) m = fmaxf(m, red_max[w]);

  // Blocks use different references, so the exponent difference is formed
  // first (exact for the largest terms) instead of folded into an FMA.
  const unsigned live = SC ? live_chunks<T, VPT, THREADS, ALIGNED, int>(vb, lim, t) : ~0u;
  float s = warp_sum(exp_sum<T, VPT, false>(raw, v, exp_ref(m), k, live));
  if (lane == 0) red_sum[warp] = s;
  __syncthreads();
  s = red_sum[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) s += red_sum[w];

  const float2 ML = exchange_merge(ex, m, s, csize, crank, k);
  store_chunks<T, VPT, THREADS, ALIGNED, int, SC>(yr, vb, ve, cols, t, v, rescale(m, ML.x, k) * __frcp_rn(ML.y),
                                                  sc.skip_masked ? lim : cols);
}

// ---------------------------------------------------------------- two-phase path

__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2, float k) {
  const float M = fmaxf(m, m2);
  l = l * rescale(m, M, k) + l2 * rescale(m2, M, k);
  m = M;
}

// Streaming pass 1 over vectors [vb, ve) of a row: running (m, l) per thread
// (the online recurrence of lecture 6, section 7.2), chunk by chunk.
// MASK: only elements before lim count; chunks wholly after it are skipped.
template <typename T, int THREADS, int VPT, bool ALIGNED, bool MASK>
__device__ __forceinline__ void stream_stats(const T* xr, size_t vb, size_t ve, size_t cols, size_t lim, int t,
                                             float k, float& m, float& l) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int E = VPT * VEC;
  constexpr size_t STEP = static_cast<size_t>(THREADS) * VPT;
  if constexpr (MASK) ve = imin(ve, (lim + VEC - 1) / VEC);
  for (size_t c = vb; c < ve; c += STEP) {
    uint4 raw[VPT];
    float v[E];
    load_row<T, VPT, THREADS, ALIGNED, MASK, size_t>(xr, c, ve, cols, lim, t, raw, v);
    const float mn = fmaxf(m, row_max<T, VPT>(raw, v));
    const float acc = exp_sum<T, VPT, false>(raw, v, exp_ref(mn), k);
    l = l * rescale(m, mn, k) + acc;
    m = mn;
  }
}

// Merge every thread's (m, l) of the block; all threads get the result.
// `red` holds THREADS/32 entries; the caller must not reuse it before a
// following __syncthreads.
template <int THREADS>
__device__ __forceinline__ void block_merge_ml(float& m, float& l, float2* red, float k) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    merge_ml(m, l, m2, l2, k);
  }
  if (lane == 0) red[warp] = make_float2(m, l);
  __syncthreads();
  m = red[0].x;
  l = red[0].y;
#pragma unroll
  for (int w = 1; w < THREADS / 32; ++w) merge_ml(m, l, red[w].x, red[w].y, k);
}

// Streaming pass 2 over vectors [vb, ve): y = exp(x - M) / L (MASK: 0 at
// and after lim, without loading those elements).
template <typename T, int THREADS, int VPT, bool ALIGNED, bool MASK>
__device__ __forceinline__ void stream_normalise(const T* xr, T* yr, size_t vb, size_t ve, size_t cols, size_t lim,
                                                 int t, float k, float M, float L, size_t wlim) {
  constexpr int E = VPT * Elem<T>::VEC;
  constexpr size_t STEP = static_cast<size_t>(THREADS) * VPT;
  const float r = __frcp_rn(L);
  const float ref = exp_ref(M);
  for (size_t c = vb; c < ve; c += STEP) {
    uint4 raw[VPT];
    float v[E];
    load_row<T, VPT, THREADS, ALIGNED, MASK, size_t>(xr, c, ve, cols, lim, t, raw, v);
    exp_sum<T, VPT, false>(raw, v, ref, k);
    store_chunks<T, VPT, THREADS, ALIGNED, size_t, MASK>(yr, c, ve, cols, t, v, r, wlim);
  }
}

// Held to 32 registers, four 512-thread blocks per SM instead of three: the
// streaming passes are latency-bound, and more rows in flight pay.
// Measured on B200 (fp32, L2 cleaned): 128 x 600000 165 -> 151 us, 64 x 1M
// 139 -> 132, 512 x 1M 990 -> 964.  (The split kernels, given the same
// bound, lost 2-4% on 4M- and 16M-column rows and keep the default.)
template <typename T, bool ALIGNED, bool SC>
__global__ void __launch_bounds__(kTwoPhaseThreads, 4)
    softmax_twophase_kernel(const T* x, T* y, size_t rows, size_t cols, SoftmaxScaling sc) {
  constexpr int THREADS = kTwoPhaseThreads;
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = kTwoPhaseElemsPerThread / VEC;
  __shared__ float2 red[THREADS / 32];
  __shared__ __align__(16) ClusterExchange ex;

  const int t = threadIdx.x;
  const int csize = static_cast<int>(cluster_nctarank());  // 1 without a cluster launch
  const int crank = static_cast<int>(cluster_ctarank());
  const size_t nvec = (cols + VEC - 1) / VEC;
  const size_t per = (nvec + csize - 1) / csize;
  const size_t vb = imin(nvec, static_cast<size_t>(crank) * per);
  const size_t ve = imin(nvec, vb + per);

  // one row per cluster (the host splits launches that would exceed the grid)
  const size_t row = blockIdx.x / csize;
  if (row >= rows) return;  // same for every block of the cluster
  if (csize > 1) {
    if (t == 0) exchange_init(ex);
    cluster_arrive_relaxed();
  }
  const T* xr = x + row * cols;
  T* yr = y + row * cols;
  const float k = SC ? sc.k : kLog2e;
  const size_t lim = SC ? row_limit(sc, row, cols) : cols;

  // pass 1: running (m, l) per thread, then merged over the block
  float m = -INFINITY, l = 0.0f;
  stream_stats<T, THREADS, VPT, ALIGNED, SC>(xr, vb, ve, cols, lim, t, k, m, l);
  block_merge_ml<THREADS>(m, l, red, k);

  // merge the blocks' partials across the cluster
  if (csize > 1) {
    const float2 ML = exchange_merge(ex, m, l, csize, crank, k);
    m = ML.x;
    l = ML.y;
  }

  // pass 2: y = exp(x - M) / L
  stream_normalise<T, THREADS, VPT, ALIGNED, SC>(xr, yr, vb, ve, cols, lim, t, k, m, l,
                                                 sc.skip_masked ? lim : cols);
}

// ---------------------------------------------------------------- split path

// Rows longer than a cluster holds, split over the whole grid: block b covers
// vectors [c * chunk, (c + 1) * chunk) of row b / nchunks, c = b % nchunks.
// The stats kernel writes each chunk's (max, sum) partial to the workspace;
// the normalise kernel (next on the stream) merges the row's partials with
// the running-max rule and writes exp(x - M) / L for its chunk.  Every block
// is independent (no waits), and the number of blocks does not depend on the
// number of rows.

template <typename T, bool ALIGNED, bool SC>
__global__ void __launch_bounds__(kTwoPhaseThreads)
    softmax_split_stats_kernel(const T* x, float2* ws, size_t cols, size_t chunk, unsigned nchunks,
                               SoftmaxScaling sc) {
  constexpr int THREADS = kTwoPhaseThreads;
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = kTwoPhaseElemsPerThread / VEC;
  __shared__ float2 red[THREADS / 32];
  const size_t row = blockIdx.x / nchunks;
  const size_t c = blockIdx.x % nchunks;
  const size_t nvec = (cols + VEC - 1) / VEC;
  const size_t vb = imin(nvec, c * chunk);
  const size_t ve = imin(nvec, vb + chunk);
  const float k = SC ? sc.k : kLog2e;
  const size_t lim = SC ? row_limit(sc, row, cols) : cols;
  float m = -INFINITY, l = 0.0f;
  stream_stats<T, THREADS, VPT, ALIGNED, SC>(x + row * cols, vb, ve, cols, lim, threadIdx.x, k, m, l);
  block_merge_ml<THREADS>(m, l, red, k);
  if (threadIdx.x == 0) ws[blockIdx.x] = make_float2(m, l);
}

template <typename T, bool ALIGNED, bool SC>
__global__ void __launch_bounds__(kTwoPhaseThreads)
    softmax_split_norm_kernel(const T* x, T* y, const float2* ws, size_t cols, size_t chunk,
                              unsigned nchunks, SoftmaxScaling sc) {
  constexpr int THREADS = kTwoPhaseThreads;
  constexpr int VEC = Elem<T>::VEC;
  constexpr int VPT = kTwoPhaseElemsPerThread / VEC;
  __shared__ float2 red[THREADS / 32];
  const size_t row = blockIdx.x / nchunks;
  const size_t c = blockIdx.x % nchunks;
  const size_t nvec = (cols + VEC - 1) / VEC;
  const size_t vb = imin(nvec, c * chunk);
  const size_t ve = imin(nvec, vb + chunk);
  const float k = SC ? sc.k : kLog2e;
  const size_t lim = SC ? row_limit(sc, row, cols) : cols;
  // merge the row's partials
  const float2* part = ws + row * nchunks;
  float m = -INFINITY, l = 0.0f;
  for (unsigned i = threadIdx.x; i < nchunks; i += THREADS) merge_ml(m, l, part[i].x, part[i].y, k);
  block_merge_ml<THREADS>(m, l, red, k);
  stream_normalise<T, THREADS, VPT, ALIGNED, SC>(x + row * cols, y + row * cols, vb, ve, cols, lim, threadIdx.x, k,
                                                 m, l, sc.skip_masked ? lim : cols);
}

// A wait on an mbarrier that nothing ever arrives on: every thread gives up
// after `timeout_ns` and counts itself in g_wait_timeouts.  Exercises the
// give-up path of bounded_wait without faulting or hanging anything.
__global__ void wait_selftest_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  bounded_wait(&bar, 0, timeout_ns);
}


// ---------------------------------------------------------------- launch helpers

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), size_t blocks, int threads, int cluster,
                   cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = 0;
  if (cluster > 1) {
    if (cluster > 8) {
      const cudaError_t e =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr size_t kMaxGrid = 0x7fffffffu;

template <typename T, bool ALIGNED, bool SC>
cudaError_t launch_warp(const T* xp, T* yp, size_t rows, size_t cols, int threads, int vpt, SoftmaxScaling sc,
                        cudaStream_t s) {
  const size_t rpb = static_cast<size_t>(threads) / 32;
  size_t blocks = (rows + rpb - 1) / rpb;
  if (blocks > kMaxGrid) blocks = kMaxGrid;
  const int c = static_cast<int>(cols);
  switch (vpt) {
    case 1: return launch(softmax_warp_kernel<T, 1, ALIGNED, SC>, blocks, threads, 1, s, xp, yp, rows, c, sc);
    case 2: return launch(softmax_warp_kernel<T, 2, ALIGNED, SC>, blocks, threads, 1, s, xp, yp, rows, c, sc);
    case 4: return launch(softmax_warp_kernel<T, 4, ALIGNED, SC>, blocks, threads, 1, s, xp, yp, rows, c, sc);
    case 8: return launch(softmax_warp_kernel<T, 8, ALIGNED, SC>, blocks, threads, 1, s, xp, yp, rows, c, sc);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int EPT, bool ALIGNED, bool SC>
cudaError_t launch_block_ept(const T* xp, T* yp, size_t rows, int c, size_t blocks, int threads, SoftmaxScaling sc,
                             cudaStream_t s) {
  switch (threads) {
    case 128: return launch(softmax_block_kernel<T, 128, EPT, ALIGNED, SC>, blocks, 128, 1, s, xp, yp, rows, c, sc);
    case 256: return launch(softmax_block_kernel<T, 256, EPT, ALIGNED, SC>, blocks, 256, 1, s, xp, yp, rows, c, sc);
    case 512: return launch(softmax_block_kernel<T, 512, EPT, ALIGNED, SC>, blocks, 512, 1, s, xp, yp, rows, c, sc);
    case 1024:
      return launch(softmax_block_kernel<T, 1024, EPT, ALIGNED, SC>, blocks, 1024, 1, s, xp, yp, rows, c, sc);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, bool ALIGNED, bool SC>
cudaError_t launch_block(const T* xp, T* yp, size_t rows, size_t cols, int threads, int vpt, SoftmaxScaling sc,
                         cudaStream_t s) {
  const size_t blocks = rows < kMaxGrid ? rows : kMaxGrid;
  const int c = static_cast<int>(cols);
  switch (vpt * Elem<T>::VEC) {
    case 16: return launch_block_ept<T, 16, ALIGNED, SC>(xp, yp, rows, c, blocks, threads, sc, s);
    case 32: return launch_block_ept<T, 32, ALIGNED, SC>(xp, yp, rows, c, blocks, threads, sc, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int EPT, bool ALIGNED, bool SC>
cudaError_t launch_cluster_ept(const T* xp, T* yp, size_t rows, int c, size_t blocks, int threads, int k,
                               SoftmaxScaling sc, cudaStream_t s) {
  switch (threads) {
    case 128:
      return launch(softmax_cluster_kernel<T, 128, EPT, ALIGNED, SC>, blocks, 128, k, s, xp, yp, rows, c, sc);
    case 256:
      return launch(softmax_cluster_kernel<T, 256, EPT, ALIGNED, SC>, blocks, 256, k, s, xp, yp, rows, c, sc);
    case 512:
      return launch(softmax_cluster_kernel<T, 512, EPT, ALIGNED, SC>, blocks, 512, k, s, xp, yp, rows, c, sc);
    case 1024:
      if constexpr (EPT <= 32) {
        return launch(softmax_cluster_kernel<T, 1024, EPT, ALIGNED, SC>, blocks, 1024, k, s, xp, yp, rows, c, sc);
      }
      return cudaErrorInvalidValue;  // 64 values per thread do not fit 1024 threads' registers
    default: return cudaErrorInvalidValue;
  }
}

// Cluster launches handle one row per cluster; rows beyond one grid's worth
// of clusters go to further launches.
template <typename T, bool ALIGNED, bool SC>
cudaError_t launch_cluster(const T* xp, T* yp, size_t rows, size_t cols, int threads, int vpt, int cluster,
                           SoftmaxScaling sc, cudaStream_t s) {
  const size_t cl = static_cast<size_t>(cluster);
  const size_t max_rows = kMaxGrid / cl;
  const int c = static_cast<int>(cols);
  const size_t row0 = sc.row0;
  for (size_t r0 = 0; r0 < rows; r0 += max_rows) {
    const size_t n = (rows - r0 < max_rows) ? rows - r0 : max_rows;
    const T* xs = xp + r0 * cols;
    T* ys = yp + r0 * cols;
    sc.row0 = row0 + r0;
    cudaError_t e;
    switch (vpt * Elem<T>::VEC) {
      case 16: e = launch_cluster_ept<T, 16, ALIGNED, SC>(xs, ys, n, c, n * cl, threads, cluster, sc, s); break;
      case 32: e = launch_cluster_ept<T, 32, ALIGNED, SC>(xs, ys, n, c, n * cl, threads, cluster, sc, s); break;
      case 64: e = launch_cluster_ept<T, 64, ALIGNED, SC>(xs, ys, n, c, n * cl, threads, cluster, sc, s); break;
      default: e = cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T, bool ALIGNED, bool SC>
cudaError_t launch_twophase(const T* xp, T* yp, size_t rows, size_t cols, int cluster, SoftmaxScaling sc,
                            cudaStream_t s) {
  const size_t cl = static_cast<size_t>(cluster);
  const size_t max_rows = kMaxGrid / cl;
  const size_t row0 = sc.row0;
  for (size_t r0 = 0; r0 < rows; r0 += max_rows) {
    const size_t n = (rows - r0 < max_rows) ? rows - r0 : max_rows;
    sc.row0 = row0 + r0;
    const cudaError_t e = launch(softmax_twophase_kernel<T, ALIGNED, SC>, n * cl, kTwoPhaseThreads, cluster, s,
                                 xp + r0 * cols, yp + r0 * cols, n, cols, sc);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Stats then normalise, batch by batch of rows (a batch's partials fit the
// workspace; batches run in stream order, so the workspace is reused).
template <typename T, bool ALIGNED, bool SC>
cudaError_t launch_split(const T* xp, T* yp, size_t rows, size_t cols, const SplitGeometry& g, void* ws,
                         SoftmaxScaling sc, cudaStream_t s) {
  float2* w = static_cast<float2*>(ws);
  const size_t row0 = sc.row0;
  for (size_t r0 = 0; r0 < rows; r0 += g.rows_per_launch) {
    const size_t n = (rows - r0 < g.rows_per_launch) ? rows - r0 : g.rows_per_launch;
    const size_t blocks = n * g.nchunks;
    sc.row0 = row0 + r0;
    cudaError_t e = launch(softmax_split_stats_kernel<T, ALIGNED, SC>, blocks, kTwoPhaseThreads, 1, s,
                           xp + r0 * cols, w, cols, g.chunk_vecs, g.nchunks, sc);
    if (e != cudaSuccess) return e;
    e = launch(softmax_split_norm_kernel<T, ALIGNED, SC>, blocks, kTwoPhaseThreads, 1, s, xp + r0 * cols,
               yp + r0 * cols, static_cast<const float2*>(w), cols, g.chunk_vecs, g.nchunks, sc);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T, bool ALIGNED, bool SC>
cudaError_t launch_typed(const void* x, void* y, size_t rows, size_t cols, const fk_softmax_plan& p, void* ws,
                         const SoftmaxScaling& sc, cudaStream_t s) {
  const T* xp = static_cast<const T*>(x);
  T* yp = static_cast<T*>(y);
  switch (p.path) {
    case FK_PATH_WARP: return launch_warp<T, ALIGNED, SC>(xp, yp, rows, cols, p.threads, p.vpt, sc, s);
    case FK_PATH_CTA: return launch_block<T, ALIGNED, SC>(xp, yp, rows, cols, p.threads, p.vpt, sc, s);
    case FK_PATH_CLUSTER:
      return launch_cluster<T, ALIGNED, SC>(xp, yp, rows, cols, p.threads, p.vpt, p.cluster, sc, s);
    case FK_PATH_TWOPHASE: return launch_twophase<T, ALIGNED, SC>(xp, yp, rows, cols, p.cluster, sc, s);
    case FK_PATH_SPLIT:
      return launch_split<T, ALIGNED, SC>(xp, yp, rows, cols,
                                          split_geometry(rows, cols, Elem<T>::VEC == 8 ? FK_BF16 : FK_F32), ws, sc, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t launch_dtype(const void* x, void* y, size_t rows, size_t cols, const fk_softmax_plan& p, bool aligned,
                         void* ws, const SoftmaxScaling* sc, cudaStream_t s) {
  if (sc == nullptr) {
    const SoftmaxScaling none = {kLog2e, 0, 0, 0, 0, 0, 0, 0, 0};
    return aligned ? launch_typed<T, true, false>(x, y, rows, cols, p, ws, none, s)
                   : launch_typed<T, false, false>(x, y, rows, cols, p, ws, none, s);
  }
  return aligned ? launch_typed<T, true, true>(x, y, rows, cols, p, ws, *sc, s)
                 : launch_typed<T, false, true>(x, y, rows, cols, p, ws, *sc, s);
}

}  // namespace

cudaError_t launch_softmax(const void* x, void* y, size_t rows, size_t cols, int dtype,
                           const fk_softmax_plan& plan, bool aligned, void* ws, const SoftmaxScaling* sc,
                           const DeviceInfo& dev, cudaStream_t stream) {
  (void)dev;
  if (dtype == FK_F32) return launch_dtype<float>(x, y, rows, cols, plan, aligned, ws, sc, stream);
  return launch_dtype<__nv_bfloat16>(x, y, rows, cols, plan, aligned, ws, sc, stream);
}

cudaError_t read_wait_timeouts(unsigned* out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_wait_timeouts, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof(unsigned));
  }
  return e;
}

cudaError_t launch_wait_selftest(unsigned timeout_us, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError();
}

}  // namespace fk
