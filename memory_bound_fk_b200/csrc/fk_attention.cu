// fk_attention.cu -- attention forward on the sm_100a tensor cores:
// O = softmax(scale Q K^T, causal mask) V, the computation Flash Attention
// tiles (lecture 6, "GPU Kernels and Triton", sections 7.3 and 8): for one
// block of queries, loop over blocks of keys, keep a running row max m and
// sum l, rescale the output accumulator when m grows, and divide by l at the
// end -- the online recurrence of section 7.2 -- so S and P never reach HBM.
//
// One CTA of 384 threads per (pair of 128-query blocks, batch*head): one
// softmax warpgroup per query tile (thread r owns row r of its tile: TMEM
// lane r, the whole 128-key row of S in registers, so the row max needs no
// exchange), and a producer warpgroup whose first warp issues every MMA and
// whose second issues every TMA load (the other two idle).  setmaxnreg moves
// registers from the producer warpgroup to the softmax warpgroups.  Each
// K_j, V_j tile brought into shared memory serves both query tiles.
//   S_i   (128 x 128 fp32, TMEM columns 256 i ..)        = Q_i K_j^T   (tcgen05.mma, A and B in smem)
//   P_i   (128 x 128 bf16, over the first 64 columns of S_i)            (written by the softmax threads)
//   O_i   (128 x D   fp32, TMEM columns 256 i + 128 ..) += P_i V_j     (tcgen05.mma, A in TMEM)
// Q, K_j, V_j arrive by TMA in 128-byte-swizzled tiles, two buffers each for
// K and V.  The MMA thread issues in the order S_0,0 S_1,0 | O_0,j S_0,j+1 |
// O_1,j S_1,j+1 | ..., so the tensor cores work on one tile while the other
// tile's warpgroup computes its exponentials; after the last MMA that reads
// K_j (or V_j) it commits to that buffer's "free" barrier, on which the load
// thread waits before it refills the buffer.  The MMAs of one thread complete
// in issue order (tcgen05.commit reports everything issued before it), so
// "S_i,j+1 done" also means "O_i,j done and P_i,j read".  Every mbarrier
// wait is bounded (1 s); a wait that gives up is counted, the whole CTA
// stops, waits (again bounded) for its copies and MMAs in flight, frees its
// TMEM and returns.
//
// The running max is lazy (the rescaling rule of the online softmax holds
// for any reference value, not only the true max): a row's reference moves
// only when the block max exceeds it by more than 2^8, so the weights stay
// at most 256 and the O rescale -- a TMEM round trip -- is rare.
// Causal grids hand out the longest query-tile pairs first; other grids keep
// the pairs of a slice together in launch order, for L2 reuse of K and V.
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
constexpr int kAttnThreads = 3 * kAttnTileThreads;       // + the producer warpgroup
constexpr int kMmaWarp = 8, kLoadWarp = 9;               // producer warps (10, 11 idle)
constexpr int kSoftmaxRegs = 208, kProducerRegs = 88;    // setmaxnreg split of the launch's registers
constexpr int kSplitRegs = kAttnTileThreads * (2 * kSoftmaxRegs + kProducerRegs);
static_assert(kSplitRegs <= 65536, "register split above the register file");
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
  if (mbar_test_wait(bar, parity)) return true;
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

// max(a, b, c) in one instruction (sm_100); a NaN operand is ignored, as by
// fmaxf.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fp32 lanes per instruction (sm_100 packed arithmetic), each rounded as
// the scalar operation would be.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// One key block j of a softmax thread (row r of its tile; S in TMEM at tS,
// O at tO): the row max, the lazy reference m (moved only when the block's
// max exceeds it by more than kLazyRescale), p = 2^(s scale log2e - m)
// written as bf16 over the first 64 columns of S, the running sum, and O
// rescaled when m moved.  DIAG: the causal grid's diagonal block, whose keys
// after the query are set to -inf in registers first (exp gives 0), so the
// other blocks carry no per-element mask.
template <bool DIAG>
__device__ __forceinline__ void softmax_block(uint32_t tS, uint32_t tO, int d_cols, int r, int j, float scale_log2,
                                              float& m_i, float& l_i) {
  tc::fence_after_sync();
  uint32_t sr[128];
#pragma unroll
  for (int c = 0; c < 4; ++c) tc::tmem_ld32_async(tS + c * 32, sr + c * 32);
  tc::tmem_wait_ld();
  if (DIAG) {
#pragma unroll
    for (int i = 0; i < 128; ++i) sr[i] = (i > r) ? 0xff800000u : sr[i];
  }
  // eight running maxima, two values folded in per three-input max
  float mx8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[8 + k]));
#pragma unroll
  for (int i = 16; i < 128; i += 16)  // values i .. i + 15 (the last group ends at 127)
#pragma unroll
    for (int k = 0; k < 8; ++k) mx8[k] = max3(mx8[k], __uint_as_float(sr[i + k]), __uint_as_float(sr[i + 8 + k]));
  const float mx = max3(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])) *
                   scale_log2;
  const bool upd = mx > m_i + kLazyRescale;  // always for the first block (m_i = -inf)
  const float m_new = upd ? mx : m_i;
  const float corr = upd ? ex2_ftz(m_i - m_new) : 1.0f;
  const float2 k2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_new, -m_new);
  float2 sum4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sum4[i] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 x =
          ffma2(make_float2(__uint_as_float(sr[c * 16 + i]), __uint_as_float(sr[c * 16 + i + 1])), k2, nm2);
      const float2 p = make_float2(ex2_ftz(x.x), ex2_ftz(x.y));
      sum4[(i >> 1) & 3] = fadd2(sum4[(i >> 1) & 3], p);
      w[i >> 1] = pack_bf16x2(p.x, p.y);
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
  const float2 s2 = fadd2(fadd2(sum4[0], sum4[1]), fadd2(sum4[2], sum4[3]));
  l_i = fmaf(l_i, corr, s2.x + s2.y);
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

// The units of work, a pair of 128-query tiles of one slice, in the order
// they are handed out: causal grids take the longest pairs (most key
// blocks) first, across all slices; other grids keep the pairs of a slice
// together, so that its K/V tiles are read from HBM once and then hit L2.
// Each block is persistent and takes the units blockIdx.x, then
// 2 G - 1 - blockIdx.x, then 2 G + blockIdx.x, ... (G blocks): a serpentine
// that balances the decreasing causal unit lengths across blocks, and lets
// a block start its next unit's loads while the current one finishes.
//
// Equal units (the non-causal grid) leave the last round part-empty: 512
// units on 148 blocks make 3.46 rounds, and the blocks with a fourth unit set
// the time.  When the last round's units are at most half the blocks, each
// of them is split into two halves of its key blocks, run by two blocks;
// the online recurrence of section 7.2 merges the halves exactly (the same
// rule that merges key blocks), see merge_halves.
struct AttnWork {
  int u;     // the unit; -1: no more work for this block
  int half;  // -1: the whole unit; 0 / 1: the first / second half of its key blocks
};

struct AttnUnits {
  int t, bh;       // keys (and queries) per slice, slices
  int nfull;       // units handed out whole; the rest (nsplit) are split in halves
  int nsplit;
  bool causal;
  __device__ __forceinline__ int nq() const { return t / 128; }
  __device__ __forceinline__ int npair() const { return (nq() + 1) / 2; }
  __device__ __forceinline__ AttnWork work(int round) const {
    const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    const int w = (round & 1) ? g - 1 - b : b;
    const int base = round * g;
    if (nsplit > 0 && base >= nfull) {  // the last round: half units
      if (base > nfull || w >= 2 * nsplit) return AttnWork{-1, -1};
      return AttnWork{nfull + w / 2, w & 1};
    }
    const int u = base + w;
    return AttnWork{u < bh * npair() ? u : -1, -1};
  }
  __device__ __forceinline__ int slice(int u) const { return causal ? u % bh : u / npair(); }
  __device__ __forceinline__ int pair(int u) const { return causal ? npair() - 1 - u / bh : u % npair(); }
  // key blocks of query tile i of unit u (0: the tile is absent, when nq is
  // odd and this is the last pair)
  __device__ __forceinline__ int nkv(int u, int i) const {
    const int qb = 2 * pair(u) + i;
    return qb < nq() ? (causal ? qb + 1 : nq()) : 0;
  }
  // first key block and key blocks of query tile i for a piece of work
  // (halves are made only of non-causal units, whose tiles see every key)
  __device__ __forceinline__ int key0(const AttnWork& wk) const { return wk.half == 1 ? nq() / 2 : 0; }
  __device__ __forceinline__ int nkv(const AttnWork& wk, int i) const {
    const int n = nkv(wk.u, i);
    if (wk.half < 0 || n == 0) return n;
    return wk.half == 0 ? nq() / 2 : nq() - nq() / 2;
  }
};

// Scratch of the split units (global memory): per split unit, half and
// query tile, every row's unnormalised O (fp32) and its (reference max m,
// sum l), and per split unit and tile a counter of the halves that finished.
struct AttnSplitScratch {
  float* o;        // [nsplit][2 halves][2 tiles][D / 4 column quads][128 rows][4]: a warp's
                   // 32 rows of one quad are 512 contiguous bytes
  float2* ml;      // [nsplit][2 halves][2 tiles][128 rows]
  unsigned* done;  // [nsplit][2 tiles], zero at launch
};

// Named barrier 1 + i for the 128 threads of softmax warpgroup i (barrier 0
// is the block-wide one).
__device__ __forceinline__ void warpgroup_bar(int i) {
  if (i == 0)
    asm volatile("bar.sync 1, 128;" ::: "memory");
  else
    asm volatile("bar.sync 2, 128;" ::: "memory");
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attention_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, __nv_bfloat16* __restrict__ out, int t, int bh,
                         int nfull, int nsplit, AttnSplitScratch split, float scale_log2) {
  constexpr int KC = D / 64;                     // 64-column chunks of a head row
  constexpr uint32_t TILE = KC * kChunkBytes;    // bytes of a 128 x D tile
  constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, 128, false);
  constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(128, D, true);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_qfree, bar_k[2], bar_v[2], bar_kfree[2], bar_vfree[2], bar_s[2], bar_p[2],
      bar_o[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int split_flag[2];  // per softmax warpgroup: decisions taken once for its 128 threads

  // Q0 | Q1 | K0 | K1 | V0 | V1, every tile 1024-byte aligned (addressed by
  // offset: arrays of pointers indexed at run time would live in local memory)
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  auto sQ = [&](int i) { return base + i * TILE; };
  auto sK = [&](int b) { return base + (2 + b) * TILE; };
  auto sV = [&](int b) { return base + (4 + b) * TILE; };

  const int tid = threadIdx.x, warp = tid >> 5;
  const AttnUnits units{t, bh, nfull, nsplit, CAUSAL};
  volatile int* abort = &abort_flag;

  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_qfree, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k[i], 1);
      mbar_init(&bar_v[i], 1);
      mbar_init(&bar_kfree[i], 1);
      mbar_init(&bar_vfree[i], 1);
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_o[i], 1);
      mbar_init(&bar_p[i], kAttnTileThreads / 32);  // one arrival per softmax warp
    }
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;

  // Barrier phases run on from one unit to the next: Q and its "free"
  // barrier complete once per unit, the K and V buffers are filled by one
  // tile counter g across units (tile g in buffer g % 2), and S, P and O of
  // each query tile count their phases across units.
  if (warp >= 2 * kAttnTileThreads / 32) {
    // ------------------------------------------------ producer warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs) : "memory");
    if (warp == kLoadWarp && (tid & 31) == 0) {
      // ---- TMA loads: per unit, Q once the tensor cores are done with the
      // previous unit's S products, then K_g and V_g into buffer g % 2 once
      // the MMAs that read tile g - 2 have completed
      int g = 0, nk = 0, nv = 0;  // K/V tiles issued (counted across units)
      int nql = 0;                // Q loads issued
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const AttnWork wk = units.work(round);
        if (wk.u < 0) break;
        const int nkv0 = units.nkv(wk, 0), nkv1 = units.nkv(wk, 1);
        const int nmax = nkv0 > nkv1 ? nkv0 : nkv1, ntiles = nkv1 > 0 ? 2 : 1;
        const int row0 = units.slice(wk.u) * t;  // first row of the slice in the [bh * t, D] view
        const int krow0 = row0 + units.key0(wk) * kAttnBlock;
        const int pair = units.pair(wk.u);
        if (round > 0 && !attn_wait(&bar_qfree, (round - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bar_q, ntiles * TILE);
        for (int i = 0; i < ntiles; ++i) {
#pragma unroll
          for (int c = 0; c < KC; ++c)
            tc::tma_load_2d(sQ(i) + c * kChunkBytes, &tmq, &bar_q, c * 64, row0 + (2 * pair + i) * kAttnBlock);
        }
        nql = round + 1;
        for (int j = 0; j < nmax; ++j, ++g) {
          const int b = g & 1;
          if (g >= 2 && !attn_wait(&bar_kfree[b], ((g - 2) >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k[b], TILE);
#pragma unroll
          for (int c = 0; c < KC; ++c)
            tc::tma_load_2d(sK(b) + c * kChunkBytes, &tmk, &bar_k[b], c * 64, krow0 + j * 128);
          nk = g + 1;
          if (g >= 2 && !attn_wait(&bar_vfree[b], ((g - 2) >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v[b], TILE);
#pragma unroll
          for (int c = 0; c < KC; ++c)
            tc::tma_load_2d(sV(b) + c * kChunkBytes, &tmv, &bar_v[b], c * 64, krow0 + j * 128);
          nv = g + 1;
        }
      }
      // copies in flight land before the CTA exits.  Q is reloaded only after
      // the MMA warp has seen the previous Q land, and a K/V buffer is refilled
      // only after it has seen that buffer's previous load land, so only the
      // last Q load and the last load into each buffer can be pending.
      if (nql > 0) drain_wait(&bar_q, (nql - 1) & 1);
      for (int j = nk > 2 ? nk - 2 : 0; j < nk; ++j) drain_wait(&bar_k[j & 1], (j >> 1) & 1);
      for (int j = nv > 2 ? nv - 2 : 0; j < nv; ++j) drain_wait(&bar_v[j & 1], (j >> 1) & 1);
    } else if (warp == kMmaWarp && (tid & 31) == 0) {
      // ---- MMA issue
      int k_wt = 0, v_wt = 0;  // K_0 .. K_k_wt-1, V_0 .. V_v_wt-1 (across units) seen in shared memory
      auto wait_k = [&](int g) {
        if (g < k_wt) return true;
        if (!attn_wait(&bar_k[g & 1], (g >> 1) & 1, abort)) return false;
        k_wt = g + 1;
        return true;
      };
      auto wait_v = [&](int g) {
        if (g < v_wt) return true;
        if (!attn_wait(&bar_v[g & 1], (g >> 1) & 1, abort)) return false;
        v_wt = g + 1;
        return true;
      };
      // shared-memory descriptors, low words (the high words are constants):
      // one per buffer, stepped through a tile by constant offsets
      constexpr uint32_t HI = tc::smem_desc_hi(1024);
      const uint32_t dq0 = tc::smem_desc_lo(smem_addr(sQ(0)), 16);
      const uint32_t dk0 = tc::smem_desc_lo(smem_addr(sK(0)), 16);
      const uint32_t dv0 = tc::smem_desc_lo(smem_addr(sV(0)), kChunkBytes);
      int np[2] = {0, 0};  // P arrivals waited for, per query tile (across units)
      int g0 = 0;          // tile counter of the unit's first K/V tile
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const AttnWork wk = units.work(round);
        if (wk.u < 0) break;
        const int nkv0 = units.nkv(wk, 0), nkv1 = units.nkv(wk, 1);
        const int nmax = nkv0 > nkv1 ? nkv0 : nkv1, ntiles = nkv1 > 0 ? 2 : 1;
        int s_left = nkv0 + nkv1;  // S products of the unit still to issue
        auto last = [&](int j) { return j < nkv1 ? 1 : 0; };  // the tile that reads K_j and V_j last
        // S_i = Q_i K_j^T into TMEM columns 256 i ..; after the unit's last
        // one, Q may be reloaded once it completes
        auto issue_s = [&](int i, int j) {
          const uint32_t dq = dq0 + i * (TILE >> 4), dk = dk0 + ((g0 + j) & 1) * (TILE >> 4);
          const uint32_t ts = tmem + i * 256;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = ((ks / 4) * kChunkBytes + (ks % 4) * 32) >> 4;
            tc::mma_bf16(ts, tc::desc_join(dq + off, HI), tc::desc_join(dk + off, HI), IDESC_S, ks > 0 ? 1u : 0u);
          }
          tc::mma_commit(&bar_s[i]);
          if (i == last(j)) tc::mma_commit(&bar_kfree[(g0 + j) & 1]);
          if (--s_left == 0) tc::mma_commit(&bar_qfree);
        };
        // O_i += P_i V_j: P_i (TMEM, 8 columns per 16 keys), V_j MN-major in smem.
        // The unit's first one overwrites O_i, which the previous unit's
        // epilogue has read by then: its softmax warpgroup arrives on P_i only
        // after that epilogue.
        auto issue_o = [&](int i, int j) {
          const uint32_t dv = dv0 + ((g0 + j) & 1) * (TILE >> 4);
          const uint32_t to = tmem + i * 256 + 128, tp = tmem + i * 256;
          const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
          for (int ks = 0; ks < kAttnBlock / 16; ++ks)
            tc::mma_bf16_ts(to, tp + ks * 8, tc::desc_join(dv + ((ks * 2048) >> 4), HI), IDESC_O, ks > 0 ? 1u : acc0);
          if (i == last(j)) tc::mma_commit(&bar_vfree[(g0 + j) & 1]);
        };

        ok = attn_wait(&bar_q, round & 1, abort) && wait_k(g0);
        if (!ok) break;
        tc::fence_after_sync();
        for (int i = 0; i < ntiles; ++i) issue_s(i, 0);
        for (int j = 0; ok && j < nmax; ++j) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int nkv_i = i == 0 ? nkv0 : nkv1;
            if (!ok || j >= nkv_i) continue;
            // the tiles first (long since loaded: their loads wait only on
            // MMAs already issued), then softmax i's block j: P_i,j written,
            // O_i rescaled.  The two MMA groups then go out back to back.
            ok = wait_v(g0 + j) && (j + 1 >= nkv_i || wait_k(g0 + j + 1)) && attn_wait(&bar_p[i], np[i] & 1, abort);
            if (!ok) break;
            ++np[i];
            tc::fence_after_sync();
            issue_o(i, j);
            if (j + 1 < nkv_i) {
              issue_s(i, j + 1);
            } else {
              tc::mma_commit(&bar_o[i]);
            }
          }
        }
        g0 += nmax;
      }
      // every MMA completes before the CTA exits
      tc::mma_commit(&bar_drain);
      drain_wait(&bar_drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax warpgroup i: query tile 2 pair + i of each unit
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs) : "memory");
    const int i = warp >> 2;
    const int r = ((warp & 3) << 5) | (tid & 31);
    const uint32_t lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane + i * 256, tO = tS + 128;
    int ns = 0, no = 0;  // S and O phases waited for (across units)
    for (int round = 0;; ++round) {
      const AttnWork wk = units.work(round);
      if (wk.u < 0) break;
      const int qb = 2 * units.pair(wk.u) + i;
      const int nkv_i = units.nkv(wk, i);
      float m_i = -INFINITY, l_i = 0.0f;
      for (int j = 0; j < nkv_i; ++j, ++ns) {
        attn_wait(&bar_s[i], ns & 1, abort);
        if (!__any_sync(0xffffffffu, *abort)) {
          if (CAUSAL && j == qb)
            softmax_block<true>(tS, tO, D, r, j, scale_log2, m_i, l_i);
          else
            softmax_block<false>(tS, tO, D, r, j, scale_log2, m_i, l_i);
        }
        // each thread's P stores are complete (tcgen05.wait::st); one lane
        // per warp arrives once the warp has synchronised
        tc::fence_before_sync();
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(&bar_p[i]);
      }
      if (nkv_i == 0) continue;
      attn_wait(&bar_o[i], no & 1, abort);
      ++no;
      // row r of the tile in the output
      uint4* dst =
          reinterpret_cast<uint4*>(out + (static_cast<size_t>(units.slice(wk.u)) * t + qb * kAttnBlock + r) * D);
      if (wk.half < 0) {
        if (!__any_sync(0xffffffffu, *abort)) {
          tc::fence_after_sync();
          // O / l, rounded to bf16
          const float inv = 1.0f / l_i;
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
      } else if constexpr (!CAUSAL) {
        // Half of a split unit (non-causal grids only).  Both halves store their rows' unnormalised
        // O and (m, l); the half that finishes second (by an atomic count
        // per unit and tile, taken after a fence) merges the other's with
        // its own and writes the output.  Nothing waits on the other block.
        // The warpgroup's 128 threads take each decision together (its named
        // barrier), so that all of them pass the same barriers.
        warpgroup_bar(i);
        if (r == 0) split_flag[i] = *abort;
        warpgroup_bar(i);
        if (!split_flag[i]) {
          const int su = wk.u - nfull;
          const size_t tmine = static_cast<size_t>(su * 2 + wk.half) * 2 + i;
          const size_t tother = static_cast<size_t>(su * 2 + (1 - wk.half)) * 2 + i;
          const size_t mine = tmine * kAttnBlock + r, other = tother * kAttnBlock + r;
          tc::fence_after_sync();
          float4* po = reinterpret_cast<float4*>(split.o) + tmine * kAttnBlock * (D / 4) + r;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tc::tmem_ld32(tO + c * 32, v);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              po[(c * 8 + q) * kAttnBlock] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
          split.ml[mine] = make_float2(m_i, l_i);
          __threadfence();
          warpgroup_bar(i);
          if (r == 0) split_flag[i] = static_cast<int>(atomicAdd(&split.done[su * 2 + i], 1u));
          warpgroup_bar(i);
          if (split_flag[i] == 1) {
            __threadfence();
            // the other half's (m, l) and O, read through L2 (written by
            // another SM), all of the row's loads in flight at once
            const float4* oo = reinterpret_cast<const float4*>(split.o) + tother * kAttnBlock * (D / 4) + r;
            const float2 mlo = __ldcg(split.ml + other);
            float4 wo[D / 4];
#pragma unroll
            for (int q = 0; q < D / 4; ++q) wo[q] = __ldcg(oo + q * kAttnBlock);
            const float M = fmaxf(m_i, mlo.x);
            const float fa = (m_i == M) ? 1.0f : ex2_ftz(m_i - M);
            const float fb = (mlo.x == M) ? 1.0f : ex2_ftz(mlo.x - M);
            const float inv = 1.0f / fmaf(l_i, fa, mlo.y * fb);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float v[32];
              tc::tmem_ld32(tO + c * 32, v);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 w = wo[c * 8 + q];
                v[4 * q] = fmaf(v[4 * q], fa, w.x * fb) * inv;
                v[4 * q + 1] = fmaf(v[4 * q + 1], fa, w.y * fb) * inv;
                v[4 * q + 2] = fmaf(v[4 * q + 2], fa, w.z * fb) * inv;
                v[4 * q + 3] = fmaf(v[4 * q + 3], fa, w.w * fb) * inv;
              }
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[c * 4 + q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                            pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                                            pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
            }
          }
        }
      }
      // the next unit's first O product overwrites O: this warpgroup's
      // tcgen05.ld reads of it have completed (tmem_ld32 waits for them)
      // before its next arrival on P
      tc::fence_before_sync();
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

// How the units go to the persistent blocks: G blocks, the first nfull
// units whole, the remaining nsplit units (the last, part-empty round of a
// non-causal grid, when it fills at most half the blocks) in key halves.
struct AttnGrid {
  int blocks, nfull, nsplit;
};

AttnGrid attn_grid(size_t bh, size_t t, bool causal, int sm_count) {
  const size_t nq = t / kAttnBlock;
  const size_t nunits = bh * ((nq + 1) / 2);
  const size_t sms = static_cast<size_t>(sm_count);
  const size_t rounds = (nunits + sms - 1) / sms;
  const size_t last = nunits - (rounds - 1) * sms;
  if (!causal && nq >= 2 && 2 * last <= sms)
    return AttnGrid{sm_count, static_cast<int>(nunits - last), static_cast<int>(last)};
  return AttnGrid{static_cast<int>(nunits < sms ? nunits : sms), static_cast<int>(nunits), 0};
}

template <int D, bool CAUSAL>
cudaError_t launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, void* o, size_t bh,
                        size_t t, float scale_log2, int sm_count, cudaStream_t s) {
  constexpr uint32_t TILE = (D / 64) * kChunkBytes;
  const size_t smem = 6 * TILE + 1024;
  auto kernel = attention_fwd_kernel<D, CAUSAL>;
  // setmaxnreg.inc waits until the registers it asks for are free in the
  // block's pool (its threads x the registers each was launched with): the
  // split must fit that pool, or the softmax warpgroups would wait forever
  cudaFuncAttributes fa;
  cudaError_t e0 = cudaFuncGetAttributes(&fa, kernel);
  if (e0 != cudaSuccess) return e0;
  if (fa.numRegs * kAttnThreads < kSplitRegs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // persistent blocks, one per SM (the kernel holds all of an SM's tensor
  // memory), each walking its units
  const AttnGrid g = attn_grid(bh, t, CAUSAL, sm_count);
  AttnSplitScratch split = {nullptr, nullptr, nullptr};
  void* ws = nullptr;
  if (g.nsplit > 0) {
    // scratch for the split units, stream-ordered from the library's pool
    const size_t rows = static_cast<size_t>(g.nsplit) * 2 * 2 * kAttnBlock;
    const size_t o_bytes = rows * D * sizeof(float), ml_bytes = rows * sizeof(float2);
    const size_t done_bytes = static_cast<size_t>(g.nsplit) * 2 * sizeof(unsigned);
    e = workspace_alloc(&ws, o_bytes + ml_bytes + done_bytes, s);
    if (e != cudaSuccess) return e;
    char* base = static_cast<char*>(ws);
    split.o = reinterpret_cast<float*>(base);
    split.ml = reinterpret_cast<float2*>(base + o_bytes);
    split.done = reinterpret_cast<unsigned*>(base + o_bytes + ml_bytes);
    e = cudaMemsetAsync(split.done, 0, done_bytes, s);
    if (e != cudaSuccess) {
      (void)cudaFreeAsync(ws, s);
      return e;
    }
  }
  kernel<<<static_cast<unsigned>(g.blocks), kAttnThreads, smem, s>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(o), static_cast<int>(t), static_cast<int>(bh), g.nfull, g.nsplit, split,
      scale_log2);
  e = cudaGetLastError();
  if (ws != nullptr) {
    const cudaError_t f = cudaFreeAsync(ws, s);
    if (e == cudaSuccess) e = f;
  }
  return e;
}

}  // namespace

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* o, size_t bh, size_t t, int d,
                             bool causal, float scale, int sm_count, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, bh * t, d) || !make_map(&mk, k, bh * t, d) || !make_map(&mv, v, bh * t, d))
    return cudaErrorInvalidValue;
  const float sl2 = static_cast<float>(static_cast<double>(scale) * 1.44269504088896340736);
  const int sms = sm_count > 0 ? sm_count : 1;
  if (d == 64) {
    return causal ? launch_attn<64, true>(mq, mk, mv, o, bh, t, sl2, sms, stream)
                  : launch_attn<64, false>(mq, mk, mv, o, bh, t, sl2, sms, stream);
  }
  return causal ? launch_attn<128, true>(mq, mk, mv, o, bh, t, sl2, sms, stream)
                : launch_attn<128, false>(mq, mk, mv, o, bh, t, sl2, sms, stream);
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
