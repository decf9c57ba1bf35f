// fk_attention.cu -- attention forward on the sm_100a tensor cores:
// O = softmax(scale Q K^T, causal mask) V, the computation Flash Attention
// tiles (lecture 6, "GPU Kernels and Triton", sections 7.3 and 8): for one
// block of queries, loop over blocks of keys, keep a running row max m and
// sum l, rescale the output accumulator when m grows, and divide by l at the
// end -- the online recurrence of section 7.2 -- so S and P never reach HBM.
//
// One CTA of 128 threads per (128-query block, batch*head).  Thread r owns
// query row r, which is TMEM lane r of both accumulators:
//   S (128 x 128 fp32, TMEM columns 0..127)   = Q K_j^T      (tcgen05.mma)
//   O (128 x D   fp32, TMEM columns 128..)   += P_j V_j       (tcgen05.mma)
// Q, K_j, V_j arrive by TMA in 128-byte-swizzled tiles; P_j is written by the
// threads into a K-major swizzled shared-memory tile (bf16) for the second
// MMA.  One thread issues the MMAs; completion arrives on an mbarrier
// (tcgen05.commit).  Every mbarrier wait is bounded (1 s); a wait that gives
// up is counted, the whole CTA stops, frees its TMEM and returns.
//
// This first version runs the steps of one key block in sequence (TMA ->
// MMA -> softmax -> MMA); overlapping them across key blocks is the next step.
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

constexpr int kAttnThreads = 128;
constexpr int kAttnBlock = 128;                // queries per CTA = keys per step
constexpr uint32_t kChunkBytes = 128 * 128;    // 128 rows x 64 bf16 columns
constexpr uint32_t kTmemCols = 256;            // S: 128 columns, O: up to 128
constexpr uint64_t kAttnWaitNs = 1000000000ull;

__device__ __forceinline__ bool attn_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kAttnWaitNs) {
      atomicAdd(&g_attn_wait_timeouts, 1u);
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
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
  __shared__ uint64_t bar_q, bar_kv, bar_mma;
  __shared__ uint32_t tmem_slot;

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  uint8_t* sQ = base;
  uint8_t* sK = base + TILE;
  uint8_t* sV = base + 2 * TILE;
  uint8_t* sP = base + 3 * TILE;  // 2 chunks: keys 0..63, 64..127
  const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aP = smem_addr(sP);

  const int tid = threadIdx.x, warp = tid >> 5, r = tid;
  const int qblk = blockIdx.x;
  const int row0 = blockIdx.y * t + qblk * kAttnBlock;  // first query row in the [bh * t, D] view

  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_kv, 1);
    mbar_init(&bar_mma, 1);
    fence_mbarrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane, tO = tmem + lane + 128;

  if (tid == 0) {
    mbar_arrive_expect_tx(&bar_q, TILE);
#pragma unroll
    for (int c = 0; c < KC; ++c) tc::tma_load_2d(sQ + c * kChunkBytes, &tmq, &bar_q, c * 64, row0);
  }
  const int nkv = CAUSAL ? qblk + 1 : t / kAttnBlock;
  float m_i = -INFINITY, l_i = 0.0f;
  bool ok = __syncthreads_and(attn_wait(&bar_q, 0)) != 0;

  for (int j = 0; j < nkv && ok; ++j) {
    const int krow = blockIdx.y * t + j * kAttnBlock;
    if (tid == 0) {
      mbar_arrive_expect_tx(&bar_kv, 2 * TILE);
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        tc::tma_load_2d(sK + c * kChunkBytes, &tmk, &bar_kv, c * 64, krow);
        tc::tma_load_2d(sV + c * kChunkBytes, &tmv, &bar_kv, c * 64, krow);
      }
    }
    ok = __syncthreads_and(attn_wait(&bar_kv, j & 1)) != 0;
    if (!ok) break;

    // S = Q K_j^T: D/16 MMAs of K = 16, both operands K-major
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks / 4) * kChunkBytes + (ks % 4) * 32;
        tc::mma_bf16(tmem, tc::smem_desc(aQ + off, 16, 1024), tc::smem_desc(aK + off, 16, 1024), IDESC_S,
                     ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(&bar_mma);
    }
    ok = __syncthreads_and(attn_wait(&bar_mma, 0)) != 0;
    if (!ok) break;
    tc::fence_after_sync();

    // softmax step on row r: max, then p = 2^(s scale log2e - m), sum, P
    const bool diag = CAUSAL && j == qblk;
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tc::tmem_ld32(tS + c * 32, s);
#pragma unroll
      for (int i = 0; i < 32; ++i) mx = fmaxf(mx, (diag && c * 32 + i > r) ? -INFINITY : s[i]);
    }
    const float m_new = fmaxf(m_i, mx * scale_log2);
    const float corr = ex2(m_i - m_new);  // 0 for the first block (m_i = -inf)
    float sum = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tc::tmem_ld32(tS + c * 32, s);
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float p0 = (diag && c * 32 + i > r) ? 0.0f : ex2(fmaf(s[i], scale_log2, -m_new));
        const float p1 = (diag && c * 32 + i + 1 > r) ? 0.0f : ex2(fmaf(s[i + 1], scale_log2, -m_new));
        sum += p0 + p1;
        w[i / 2] = pack_bf16x2(p0, p1);
      }
      // keys c*32 .. c*32+31: chunk c/2, 16-byte units (c%2)*4 .. +3 of row r, swizzled
      uint8_t* rowp = sP + (c / 2) * kChunkBytes + r * 128;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int unit = ((c % 2) * 4 + u) ^ (r & 7);
        *reinterpret_cast<uint4*>(rowp + unit * 16) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
    }
    l_i = fmaf(l_i, corr, sum);
    m_i = m_new;

    // rescale O when the max grew (warp-uniform decision: tcgen05 ld/st are warp-wide)
    if (j > 0 && __any_sync(0xffffffffu, corr != 1.0f)) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tc::tmem_ld32(tO + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= corr;
        tc::tmem_st32(tO + c * 32, v);
      }
      tc::tmem_wait_st();
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();

    // O += P_j V_j: 8 MMAs of K = 16 keys; P K-major, V MN-major (D contiguous)
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < kAttnBlock / 16; ++ks) {
        const uint32_t offp = (ks / 4) * kChunkBytes + (ks % 4) * 32;
        tc::mma_bf16(tmem + 128, tc::smem_desc(aP + offp, 16, 1024), tc::smem_desc(aV + ks * 2048, kChunkBytes, 1024),
                     IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
      }
      tc::mma_commit(&bar_mma);
    }
    ok = __syncthreads_and(attn_wait(&bar_mma, 1)) != 0;
    tc::fence_after_sync();
  }

  if (ok) {
    // O / l, rounded to bf16, row r of the block
    const float inv = 1.0f / l_i;
    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(row0 + r) * D);
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
  const size_t smem = 3 * TILE + 2 * kChunkBytes + 1024;
  auto kernel = attention_fwd_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(t / kAttnBlock), static_cast<unsigned>(bh));
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
