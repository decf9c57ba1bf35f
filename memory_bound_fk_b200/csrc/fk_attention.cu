// fk_attention.cu -- attention forward on the sm_100a tensor cores:
// O = softmax(scale Q K^T, causal mask) V, the computation Flash Attention
// tiles (lecture 6, "GPU Kernels and Triton", sections 7.3 and 8): for one
// block of queries, loop over blocks of keys, keep a running row max m and
// sum l, rescale the output accumulator when m grows, and divide by l at the
// end -- the online recurrence of section 7.2 -- so S and P never reach HBM.
//
// One CTA of 288 threads per (128-query block, batch*head): two softmax
// warpgroups that both serve query rows 0..127 (TMEM lanes; warp w reaches
// lanes 32 (w % 4) ..), warpgroup g taking columns g*64 .. g*64+63 of S and
// its half of O, plus one producer warp.  The row max is exchanged once per
// key block through shared memory; the partial sums are added at the end.
//   S_j (128 x 128 fp32, TMEM columns (j % 2) * 128 ..) = Q K_j^T   (tcgen05.mma)
//   O   (128 x D   fp32, TMEM columns 256 ..)          += P_j V_j   (tcgen05.mma)
// Q, K_j, V_j arrive by TMA in 128-byte-swizzled tiles; P_j is written by the
// threads into a K-major swizzled shared-memory tile (bf16) for the second
// MMA.  One thread issues the MMAs; completion arrives on an mbarrier
// (tcgen05.commit).  Every mbarrier wait is bounded (1 s); a wait that gives
// up is counted, the whole CTA stops, frees its TMEM and returns.
//
// Warp specialisation: a producer warp issues every TMA load and MMA and
// talks to the softmax warps only through mbarriers (S_j ready, P_j ready,
// O_j done).  S is double-buffered in TMEM, so the tensor cores compute
// S_{j+1} while the softmax warps work on block j; K and V each have two
// buffers, refilled as soon as the MMA that read them has completed.
// Causal grids hand out the longest query blocks (most key blocks) first.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fk_common.cuh"
#include "fk_internal.h"
#include "fk_sync.cuh"
#include "fk_tc.cuh"

namespace fk {

// Number of threads whose attention mbarrier wait gave up.
__device__ unsigned int g_attn_wait_timeouts = 0;

namespace {

constexpr int kAttnSoftmaxThreads = 256;  // two warpgroups on the same 128 rows
constexpr int kAttnThreads = kAttnSoftmaxThreads + 32;  // + the producer warp
constexpr int kAttnBlock = 128;                // queries per CTA = keys per step
constexpr uint32_t kChunkBytes = 128 * 128;    // 128 rows x 64 bf16 columns
constexpr uint32_t kTmemCols = 512;            // S0, S1: 128 columns each; O: up to 128
constexpr uint64_t kAttnWaitNs = 1000000000ull;

// Bounded mbarrier wait.  A wait that gives up (1 s) is counted and raises
// the CTA's abort flag; every other wait then returns at once, and the CTA
// skips its remaining work (but not its barriers) and frees its TMEM.
__device__ __forceinline__ bool attn_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;  // suspended up to 20 us per try
    if (*abort) return false;
    if (global_ns() - t0 > kAttnWaitNs) {
      atomicAdd(&g_attn_wait_timeouts, 1u);
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Growth of a row's max (log2 units) that the running reference may lag
// behind: the exponentials are then at most 2^8, and O is rescaled only
// when the max outgrows the reference by more than that.
constexpr float kLazyRescale = 8.0f;

// One key block of a softmax warpgroup thread (row r, columns kbase ..
// kbase+63 of S_j in TMEM buffer b): the row max (exchanged with the other
// warpgroup), the reference max m (moved only when the block's max exceeds
// it by more than kLazyRescale, the same decision in both warpgroups),
// p = 2^(s scale log2e - m) written to P_j as bf16, the running sum, and O
// rescaled when m moved (after O_{j-1} completed).  diag: the causal grid's
// diagonal block, whose keys after the query are set to -inf in registers
// first (exp gives 0), so the common body carries no per-element mask.
// Every thread executes both named barriers whatever `abort` says.
template <int D>
__device__ __forceinline__ void softmax_step(uint32_t tmem, uint32_t lane, uint32_t tO, int b, int kbase, int r,
                                             int wg, int j, bool diag, uint8_t* sPb, float (*xred)[128],
                                             uint64_t* bar_o, float scale_log2, volatile int* abort, float& m_i,
                                             float& l_i) {
  uint32_t sr[64];
  if (!__any_sync(0xffffffffu, *abort)) {
    tc::fence_after_sync();
    const uint32_t tS = tmem + lane + b * 128 + kbase;
    tc::tmem_ld32_async(tS, sr);
    tc::tmem_ld32_async(tS + 32, sr + 32);
    tc::tmem_wait_ld();
    if (diag) {
#pragma unroll
      for (int i = 0; i < 64; ++i) sr[i] = (kbase + i > r) ? 0xff800000u : sr[i];
    }
    float mx8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
    for (int i = 0; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(sr[i]));
    xred[wg][r] = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                        fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
  }
  softmax_bar();  // both halves of every row's max of block j
  const float mx = fmaxf(xred[0][r], xred[1][r]) * scale_log2;
  softmax_bar();  // every read is done before the next block's writes
  const bool upd = mx > m_i + kLazyRescale;  // always for the first block (m_i = -inf)
  const float m_new = upd ? mx : m_i;
  const float corr = upd ? ex2(m_i - m_new) : 1.0f;
  // P_j's buffer was last read by O_{j-2}
  if (j >= 2) attn_wait(&bar_o[b], ((j - 2) >> 1) & 1, abort);
  if (!__any_sync(0xffffffffu, *abort)) {
    float sum8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sum8[i] = 0.0f;
    uint8_t* rowp = sPb + wg * kChunkBytes + r * 128;  // this warpgroup's keys: chunk wg of P_j
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const int k0 = c * 32 + i;
        const float p0 = ex2(fmaf(__uint_as_float(sr[k0]), scale_log2, -m_new));
        const float p1 = ex2(fmaf(__uint_as_float(sr[k0 + 1]), scale_log2, -m_new));
        sum8[(i >> 1) & 7] += p0 + p1;
        w[i / 2] = pack_bf16x2(p0, p1);
      }
      // keys kbase + c*32 .. +31: 16-byte units c*4 .. c*4+3 of row r, swizzled
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int unit = (c * 4 + u) ^ (r & 7);
        *reinterpret_cast<uint4*>(rowp + unit * 16) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
    }
    l_i = fmaf(l_i, corr, ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7])));
    m_i = m_new;
  }
  // O rescale (rare): O_{j-1} must be complete first
  if (j > 0 && __any_sync(0xffffffffu, upd)) {
    attn_wait(&bar_o[(j - 1) & 1], ((j - 1) >> 1) & 1, abort);
    if (!__any_sync(0xffffffffu, *abort)) {
      tc::fence_after_sync();
      uint32_t ov[D / 2];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tc::tmem_ld32_async(tO + c * 32, ov + c * 32);
      tc::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(ov[c * 32 + i]) * corr;
        tc::tmem_st32(tO + c * 32, v);
      }
      tc::tmem_wait_st();
    }
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attention_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, __nv_bfloat16* __restrict__ out, int t,
                         float scale_log2) {
  constexpr int KC = D / 64;                     // 64-column chunks of a head row
  constexpr uint32_t TILE = KC * kChunkBytes;    // bytes of a 128 x D tile
  constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, 128, false);
  constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(128, D, true);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_k[2], bar_v[2], bar_s[2], bar_o[2], bar_p[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  // per-warpgroup row maxima of a key block; at the end, the row sums (the
  // CTA fits the 227 KB of shared memory with ~0.9 KB to spare at D = 128)
  __shared__ float xred[2][128];

  // Q | K0 | K1 | V0 | V1 | P0 | P1, every tile 1024-byte aligned
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  uint8_t* sQ = base;
  uint8_t* sK[2] = {base + TILE, base + 2 * TILE};
  uint8_t* sV[2] = {base + 3 * TILE, base + 4 * TILE};
  uint8_t* sP[2] = {base + 5 * TILE, base + 5 * TILE + 2 * kChunkBytes};  // 2 chunks each: keys 0..63, 64..127
  const uint32_t aQ = smem_addr(sQ);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int slice = blockIdx.x;
  const int nq = static_cast<int>(gridDim.y);
  const int qblk = CAUSAL ? nq - 1 - static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y);
  const int row0 = slice * t + qblk * kAttnBlock;  // first query row in the [bh * t, D] view
  const int nkv = CAUSAL ? qblk + 1 : t / kAttnBlock;
  volatile int* abort = &abort_flag;

  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k[i], 1);
      mbar_init(&bar_v[i], 1);
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_o[i], 1);
      mbar_init(&bar_p[i], kAttnSoftmaxThreads);
    }
    abort_flag = 0;
    fence_mbarrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;  // S0 | S1 | O

  if (warp == kAttnSoftmaxThreads / 32) {
    // ------------------------------------------------ producer warp: TMA and MMA issue
    if ((tid & 31) == 0) {
      auto load_k = [&](int j) {
        const int b = j & 1;
        mbar_arrive_expect_tx(&bar_k[b], TILE);
#pragma unroll
        for (int c = 0; c < KC; ++c)
          tc::tma_load_2d(sK[b] + c * kChunkBytes, &tmk, &bar_k[b], c * 64, slice * t + j * 128);
      };
      auto load_v = [&](int j) {
        const int b = j & 1;
        mbar_arrive_expect_tx(&bar_v[b], TILE);
#pragma unroll
        for (int c = 0; c < KC; ++c)
          tc::tma_load_2d(sV[b] + c * kChunkBytes, &tmv, &bar_v[b], c * 64, slice * t + j * 128);
      };
      // S_j = Q K_j^T into TMEM columns (j % 2) * 128
      auto issue_s = [&](int j) {
        const int b = j & 1;
        if (!attn_wait(&bar_k[b], (j >> 1) & 1, abort)) return;
        tc::fence_after_sync();
        const uint32_t aK = smem_addr(sK[b]);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kChunkBytes + (ks % 4) * 32;
          tc::mma_bf16(tmem + b * 128, tc::smem_desc(aQ + off, 16, 1024), tc::smem_desc(aK + off, 16, 1024),
                       IDESC_S, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bar_s[b]);
      };
      mbar_arrive_expect_tx(&bar_q, TILE);
#pragma unroll
      for (int c = 0; c < KC; ++c) tc::tma_load_2d(sQ + c * kChunkBytes, &tmq, &bar_q, c * 64, row0);
      load_k(0);
      load_v(0);
      if (nkv > 1) {
        load_k(1);
        load_v(1);
      }
      if (attn_wait(&bar_q, 0, abort)) issue_s(0);
      for (int j = 0; j < nkv && !*abort; ++j) {
        const int b = j & 1;
        // S_{j+1}: its TMEM buffer was last read by softmax j - 1 (bar_p below)
        if (j + 1 < nkv) issue_s(j + 1);
        // K_j consumed once S_j is done: refill with K_{j+2}
        if (!attn_wait(&bar_s[b], (j >> 1) & 1, abort)) break;
        if (j + 2 < nkv) load_k(j + 2);
        // softmax j done: P_j written, S_j read, O rescaled if needed (two
        // barriers: without a rescale, softmax j+1 may finish before this
        // wait, but softmax j+2 needs S_{j+2}, issued after it)
        if (!attn_wait(&bar_p[b], (j >> 1) & 1, abort)) break;
        if (!attn_wait(&bar_v[b], (j >> 1) & 1, abort)) break;
        tc::fence_after_sync();
        const uint32_t aV = smem_addr(sV[b]), aP = smem_addr(sP[b]);
#pragma unroll
        for (int ks = 0; ks < kAttnBlock / 16; ++ks) {
          const uint32_t offp = (ks / 4) * kChunkBytes + (ks % 4) * 32;
          tc::mma_bf16(tmem + 256, tc::smem_desc(aP + offp, 16, 1024),
                       tc::smem_desc(aV + ks * 2048, kChunkBytes, 1024), IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc::mma_commit(&bar_o[b]);
        // V_{j+1} goes to the buffer of V_{j-1}, free once O_{j-1} is done
        if (j >= 1 && j + 1 < nkv) {
          if (!attn_wait(&bar_o[(j - 1) & 1], ((j - 1) >> 1) & 1, abort)) break;
          load_v(j + 1);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax warpgroups
    // Both warpgroups serve query rows 0..127 (TMEM lanes; warp w reaches
    // lanes 32 (w % 4) ..); warpgroup g takes S columns g*64 .. g*64+63 and
    // O columns g*D/2 .. .  Every thread executes every named barrier and
    // every arrival, whatever happens, so no barrier can strand a warp.
    const int wg = warp >> 2;
    const int r = ((warp & 3) << 5) | (tid & 31);
    const uint32_t lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane + 256 + wg * (D / 2);
    const int kbase = wg * 64;
    float m_i = -INFINITY, l_i = 0.0f;
    for (int j = 0; j < nkv; ++j) {
      const int b = j & 1;
      const bool diag = CAUSAL && j == qblk;
      attn_wait(&bar_s[b], (j >> 1) & 1, abort);
      // the causal mask only touches the diagonal block: the other blocks
      // take the unmasked body (no per-element tests)
      softmax_step<D>(tmem, lane, tO, b, kbase, r, wg, j, diag, sP[b], xred, bar_o, scale_log2, abort, m_i, l_i);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&bar_p[b]);
    }
    attn_wait(&bar_o[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1, abort);
    xred[wg][r] = l_i;  // the last reads of the maxima were before the last named barrier
    softmax_bar();
    if (!__any_sync(0xffffffffu, *abort)) {
      tc::fence_after_sync();
      // O / l, rounded to bf16: row r, this warpgroup's half of the columns
      const float inv = 1.0f / (xred[0][r] + xred[1][r]);
      uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(row0 + r) * D + wg * (D / 2));
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        float v[32];
        tc::tmem_ld32(tO + c * 32, v);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[c * 4 + q] = make_uint4(pack_bf16x2(v[8 * q] * inv, v[8 * q + 1] * inv),
                                      pack_bf16x2(v[8 * q + 2] * inv, v[8 * q + 3] * inv),
                                      pack_bf16x2(v[8 * q + 4] * inv, v[8 * q + 5] * inv),
                                      pack_bf16x2(v[8 * q + 6] * inv, v[8 * q + 7] * inv));
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side

using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                     const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled encode_fn() {
  static PFN_encodeTiled fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      (void)cudaGetLastError();
      return static_cast<PFN_encodeTiled>(nullptr);
    }
    return reinterpret_cast<PFN_encodeTiled>(p);
  }();
  return fn;
}

// [rows, d] bf16, boxes of 64 columns x 128 rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, size_t rows, int d) {
  PFN_encodeTiled f = encode_fn();
  if (f == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64, kAttnBlock};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool CAUSAL>
cudaError_t launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, void* o, size_t bh,
                        size_t t, float scale_log2, cudaStream_t s) {
  constexpr uint32_t TILE = (D / 64) * kChunkBytes;
  const size_t smem = 5 * TILE + 4 * kChunkBytes + 1024;
  auto kernel = attention_fwd_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(bh), static_cast<unsigned>(t / kAttnBlock));
  kernel<<<grid, kAttnThreads, smem, s>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(o), static_cast<int>(t),
                                          scale_log2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* o, size_t bh, size_t t, int d,
                             bool causal, float scale, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, bh * t, d) || !make_map(&mk, k, bh * t, d) || !make_map(&mv, v, bh * t, d))
    return cudaErrorInvalidValue;
  const float sl2 = static_cast<float>(static_cast<double>(scale) * 1.44269504088896340736);
  if (d == 64) {
    return causal ? launch_attn<64, true>(mq, mk, mv, o, bh, t, sl2, stream)
                  : launch_attn<64, false>(mq, mk, mv, o, bh, t, sl2, stream);
  }
  return causal ? launch_attn<128, true>(mq, mk, mv, o, bh, t, sl2, stream)
                : launch_attn<128, false>(mq, mk, mv, o, bh, t, sl2, stream);
}

cudaError_t read_attention_wait_timeouts(unsigned* out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_attn_wait_timeouts, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_attn_wait_timeouts, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace fk
