// fk_attention.cu -- attention forward on the sm_100a tensor cores:
// O = softmax(scale Q K^T, causal mask) V, the computation Flash Attention
// tiles (lecture 6, "GPU Kernels and Triton", sections 7.3 and 8): for one
// block of queries, loop over blocks of keys, keep a running row max m and
// sum l, rescale the output accumulator when m grows, and divide by l at the
// end -- the online recurrence of section 7.2 -- so S and P never reach HBM.
//
// One CTA of 288 threads per (pair of 128-query blocks, batch*head): one
// softmax warpgroup per query tile (thread r owns row r of its tile: TMEM
// lane r, the whole 128-key row of S in registers, so the row max needs no
// exchange), plus one producer warp.  Each K_j, V_j tile brought into
// shared memory serves both query tiles.
//   S_i   (128 x 128 fp32, TMEM columns 256 i ..)        = Q_i K_j^T   (tcgen05.mma, A and B in smem)
//   P_i   (128 x 128 bf16, over the first 64 columns of S_i)            (written by the softmax threads)
//   O_i   (128 x D   fp32, TMEM columns 256 i + 128 ..) += P_i V_j     (tcgen05.mma, A in TMEM)
// Q, K_j, V_j arrive by TMA in 128-byte-swizzled tiles.  One thread issues
// every MMA, in the order S_0,0 S_1,0 | O_0,j S_0,j+1 | O_1,j S_1,j+1 | ...,
// so the tensor cores work on one tile while the other tile's warpgroup
// computes its exponentials.  The MMAs of one thread complete in issue order
// (tcgen05.commit reports everything issued before it), so "S_i,j+1 done"
// also means "O_i,j done and P_i,j read".  Every mbarrier wait is bounded
// (1 s); a wait that gives up is counted, the whole CTA stops, waits (again
// bounded) for its copies and MMAs in flight, frees its TMEM and returns.
//
// The running max is lazy (the rescaling rule of the online softmax holds
// for any reference value, not only the true max): a row's reference moves
// only when the block max exceeds it by more than 2^8, so the weights stay
// at most 256 and the O rescale -- a TMEM round trip -- is rare.
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

constexpr int kAttnTileThreads = 128;                   // one softmax warpgroup per query tile
constexpr int kAttnThreads = 2 * kAttnTileThreads + 32;  // + the producer warp
constexpr int kAttnBlock = 128;                         // queries per tile = keys per step
constexpr uint32_t kChunkBytes = 128 * 128;             // 128 rows x 64 bf16 columns
constexpr uint32_t kTmemCols = 512;                     // tile i: S_i at 256 i, O_i at 256 i + 128
constexpr uint64_t kAttnWaitNs = 1000000000ull;
// Growth of a row's max (log2 units) that the running reference may lag
// behind: the weights are then at most 2^8.
constexpr float kLazyRescale = 8.0f;

// Bounded mbarrier wait.  A wait that gives up (1 s) is counted and raises
// the CTA's abort flag; every other wait then returns at once, and the CTA
// skips its remaining work (but not its arrivals) and frees its TMEM.
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

// Bounded wait that ignores the abort flag: copies and MMAs in flight when
// the CTA gives up must land before it exits.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
    if (global_ns() - t0 > kAttnWaitNs) {
      atomicAdd(&g_attn_wait_timeouts, 1u);
      return;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// One key block j of a softmax thread (row r of its tile; S in TMEM at tS,
// O at tO): the row max, the lazy reference m (moved only when the block's
// max exceeds it by more than kLazyRescale), p = 2^(s scale log2e - m)
// written as bf16 over the first 64 columns of S, the running sum, and O
// rescaled when m moved.  diag: the causal grid's diagonal block, whose keys
// after the query are set to -inf in registers first (exp gives 0), so the
// common body carries no per-element mask.
__device__ __forceinline__ void softmax_block(uint32_t tS, uint32_t tO, int d_cols, int r, int j, bool diag,
                                              float scale_log2, float& m_i, float& l_i) {
  tc::fence_after_sync();
  uint32_t sr[128];
#pragma unroll
  for (int c = 0; c < 4; ++c) tc::tmem_ld32_async(tS + c * 32, sr + c * 32);
  tc::tmem_wait_ld();
  if (diag) {
#pragma unroll
    for (int i = 0; i < 128; ++i) sr[i] = (i > r) ? 0xff800000u : sr[i];
  }
  float mx8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(sr[i]);
#pragma unroll
  for (int i = 8; i < 128; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(sr[i]));
  const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
                   scale_log2;
  const bool upd = mx > m_i + kLazyRescale;  // always for the first block (m_i = -inf)
  const float m_new = upd ? mx : m_i;
  const float corr = upd ? ex2_ftz(m_i - m_new) : 1.0f;
  float sum8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sum8[i] = 0.0f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float p0 = ex2_ftz(fmaf(__uint_as_float(sr[c * 16 + i]), scale_log2, -m_new));
      const float p1 = ex2_ftz(fmaf(__uint_as_float(sr[c * 16 + i + 1]), scale_log2, -m_new));
      sum8[i >> 1] += p0 + p1;
      w[i >> 1] = pack_bf16x2(p0, p1);
    }
    // keys 16c .. 16c+15 -> P columns 8c .. 8c+7 (x16 stores take two chunks)
    if (c & 1) {
      uint32_t w16[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        w16[i] = sr[(c - 1) * 16 + i];  // the previous chunk's packed words, parked in sr
        w16[8 + i] = w[i];
      }
      tc::tmem_st16(tS + (c - 1) * 8, w16);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) sr[c * 16 + i] = w[i];  // already consumed
    }
  }
  tc::tmem_wait_st();
  l_i = fmaf(l_i, corr, ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7])));
  m_i = m_new;
  // O rescale (rare): O_j-1 is complete, since S_j (issued after it) is
  if (j > 0 && __any_sync(0xffffffffu, upd)) {
    for (int c = 0; c < d_cols / 32; ++c) {
      float v[32];
      tc::tmem_ld32(tO + c * 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= corr;
      tc::tmem_st32(tO + c * 32, v);
    }
    tc::tmem_wait_st();
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
  __shared__ uint64_t bar_q, bar_k[2], bar_v[2], bar_s[2], bar_p[2], bar_o[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  // Q0 | Q1 | K0 | K1 | V0 | V1, every tile 1024-byte aligned
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  uint8_t* sQ[2] = {base, base + TILE};
  uint8_t* sK[2] = {base + 2 * TILE, base + 3 * TILE};
  uint8_t* sV[2] = {base + 4 * TILE, base + 5 * TILE};

  const int tid = threadIdx.x, warp = tid >> 5;
  const int slice = blockIdx.x;
  const int nq = t / kAttnBlock;
  const int npair = static_cast<int>(gridDim.y);
  const int pair = CAUSAL ? npair - 1 - static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y);
  // query tiles 2 pair and 2 pair + 1 (the second absent when nq is odd and
  // this is the last pair); key blocks per tile (0: absent)
  int nkv[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int qb = 2 * pair + i;
    nkv[i] = qb < nq ? (CAUSAL ? qb + 1 : nq) : 0;
  }
  volatile int* abort = &abort_flag;

  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k[i], 1);
      mbar_init(&bar_v[i], 1);
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_o[i], 1);
      mbar_init(&bar_p[i], kAttnTileThreads);
    }
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp == 2 * kAttnTileThreads / 32) {
    // ------------------------------------------------ producer warp: TMA and MMA issue
    if ((tid & 31) == 0) {
      const int nmax = nkv[0] > nkv[1] ? nkv[0] : nkv[1];
      const int ntiles = nkv[1] > 0 ? 2 : 1;
      const int row0 = slice * t;  // first row of this slice in the [bh * t, D] view
      int k_ld = 0, k_wt = 0, v_ld = 0, v_wt = 0;  // K_0 .. K_{k_ld-1} issued, K_0 .. K_{k_wt-1} seen
      auto load_k = [&](int j) {
        const int b = j & 1;
        mbar_arrive_expect_tx(&bar_k[b], TILE);
#pragma unroll
        for (int c = 0; c < KC; ++c) tc::tma_load_2d(sK[b] + c * kChunkBytes, &tmk, &bar_k[b], c * 64, row0 + j * 128);
        k_ld = j + 1;
      };
      auto load_v = [&](int j) {
        const int b = j & 1;
        mbar_arrive_expect_tx(&bar_v[b], TILE);
#pragma unroll
        for (int c = 0; c < KC; ++c) tc::tma_load_2d(sV[b] + c * kChunkBytes, &tmv, &bar_v[b], c * 64, row0 + j * 128);
        v_ld = j + 1;
      };
      auto wait_k = [&](int j) {
        if (j < k_wt) return true;
        if (!attn_wait(&bar_k[j & 1], (j >> 1) & 1, abort)) return false;
        k_wt = j + 1;
        return true;
      };
      auto wait_v = [&](int j) {
        if (j < v_wt) return true;
        if (!attn_wait(&bar_v[j & 1], (j >> 1) & 1, abort)) return false;
        v_wt = j + 1;
        return true;
      };
      // S_i = Q_i K_j^T into TMEM columns 256 i ..
      auto issue_s = [&](int i, int j) {
        const uint32_t aQ = smem_addr(sQ[i]), aK = smem_addr(sK[j & 1]);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kChunkBytes + (ks % 4) * 32;
          tc::mma_bf16(tmem + i * 256, tc::smem_desc(aQ + off, 16, 1024), tc::smem_desc(aK + off, 16, 1024),
                       IDESC_S, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bar_s[i]);
      };
      // O_i += P_i V_j: P_i (TMEM, 8 columns per 16 keys), V_j MN-major in smem
      auto issue_o = [&](int i, int j) {
        const uint32_t aV = smem_addr(sV[j & 1]);
#pragma unroll
        for (int ks = 0; ks < kAttnBlock / 16; ++ks)
          tc::mma_bf16_ts(tmem + i * 256 + 128, tmem + i * 256 + ks * 8,
                          tc::smem_desc(aV + ks * 2048, kChunkBytes, 1024), IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
      };

      mbar_arrive_expect_tx(&bar_q, ntiles * TILE);
      for (int i = 0; i < ntiles; ++i) {
#pragma unroll
        for (int c = 0; c < KC; ++c)
          tc::tma_load_2d(sQ[i] + c * kChunkBytes, &tmq, &bar_q, c * 64, row0 + (2 * pair + i) * kAttnBlock);
      }
      load_k(0);
      load_v(0);
      if (nmax > 1) {
        load_k(1);
        load_v(1);
      }
      const bool q_ok = attn_wait(&bar_q, 0, abort);
      bool ok = q_ok && wait_k(0);
      if (ok) {
        tc::fence_after_sync();
        for (int i = 0; i < ntiles; ++i) issue_s(i, 0);
      }
      for (int j = 0; ok && j < nmax; ++j) {
        const int last = j < nkv[1] ? 1 : 0;  // the tile that reads K_j last
        for (int i = 0; ok && i < 2; ++i) {
          if (i == last && (j + 2 < nmax || (j >= 1 && j + 1 < nmax))) {
            // refills: K_j was last read by S_last,j and V_j-1 by O_last,j-1,
            // both complete once S_last,j is.  This runs before S_last,j+1 is
            // issued, so bar_s[last] cannot be a phase further on.
            ok = attn_wait(&bar_s[last], j & 1, abort);
            if (!ok) break;
            if (j + 2 < nmax) load_k(j + 2);
            if (j >= 1 && j + 1 < nmax) load_v(j + 1);
          }
          if (j < nkv[i]) {
            // softmax i is done with block j: P_i,j written, O_i rescaled
            ok = attn_wait(&bar_p[i], j & 1, abort) && wait_v(j);
            if (!ok) break;
            tc::fence_after_sync();
            issue_o(i, j);
            if (j + 1 < nkv[i]) {
              ok = wait_k(j + 1);
              if (!ok) break;
              issue_s(i, j + 1);
            } else {
              tc::mma_commit(&bar_o[i]);
            }
          }
        }
      }
      // everything in flight lands before the CTA exits
      tc::mma_commit(&bar_drain);
      drain_wait(&bar_drain, 0);
      if (!q_ok) drain_wait(&bar_q, 0);
      for (int j = k_wt; j < k_ld; ++j) drain_wait(&bar_k[j & 1], (j >> 1) & 1);
      for (int j = v_wt; j < v_ld; ++j) drain_wait(&bar_v[j & 1], (j >> 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax warpgroup i: query tile 2 pair + i
    const int i = warp >> 2;
    const int r = ((warp & 3) << 5) | (tid & 31);
    const uint32_t lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane + i * 256, tO = tS + 128;
    const int qb = 2 * pair + i;
    float m_i = -INFINITY, l_i = 0.0f;
    for (int j = 0; j < nkv[i]; ++j) {
      attn_wait(&bar_s[i], j & 1, abort);
      if (!__any_sync(0xffffffffu, *abort)) softmax_block(tS, tO, D, r, j, CAUSAL && j == qb, scale_log2, m_i, l_i);
      tc::fence_before_sync();
      mbar_arrive(&bar_p[i]);
    }
    if (nkv[i] > 0) {
      attn_wait(&bar_o[i], 0, abort);
      if (!__any_sync(0xffffffffu, *abort)) {
        tc::fence_after_sync();
        // O / l, rounded to bf16: row r of the tile
        const float inv = 1.0f / l_i;
        uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(slice) * t + qb * kAttnBlock + r) * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
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
  const size_t smem = 6 * TILE + 1024;
  auto kernel = attention_fwd_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(bh), static_cast<unsigned>((t / kAttnBlock + 1) / 2));
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
