// fk_gelu.cu -- elementwise GELU, fused into one pass over HBM: every
// 16-byte vector (4 fp32 or 8 bf16 values) is read once and written once,
// all arithmetic in registers in fp32 (the fusion motivation of the CS336
// lecture-6 notes, kyc001.github.io, section 4.1).
//
// Two ways of moving the data, chosen by size (measured on B200, fp32, L2
// cleaned or left full of another kernel's dirty lines before each launch):
//   * when input and output together fit in L2 (and the input holds at
//     least 8 MiB; smaller arrays take one wave through registers), a
//     persistent pipeline through shared memory fed by the bulk-copy engine
//     (cp.async.bulk):
//     32 MiB in 11.5 us clean and 12.7 us after a dirty predecessor, against
//     13.5 and 17.0 us for loads and stores through registers;
//   * beyond that, one batch of two 16-byte loads per thread straight into
//     registers, which streams at the copy rate (7.0 TB/s at 1 GiB) where
//     the shared-memory pipeline reaches 6.0.
// The crossover is where input plus output stop fitting in L2 (the two tie
// at 64 MiB, 128 MiB in all).
//
// tanh form (the notes, section 4.2).  With u = sqrt(2/pi) (x + 0.044715 x^3),
//     0.5 x (1 + tanh u) = x * sigma(2u) = x / (1 + exp(-2u))
// (sigma the logistic function; 1 + tanh u = 2 sigma(2u)): one MUFU.EX2 for
// exp(-2u) = 2^(-2u log2 e) and one MUFU.RCP for the quotient, with no
// cancellation for either sign (for x < 0 the quotient is the small tail
// itself); an IEEE division here cost ~20 instructions per element and made
// the kernel issue-bound.  For large |x| the exponential overflows or
// flushes and y is -0 or x; tails of bf16 outputs are kept down to their
// smallest subnormal, 2^-133, by an exponent offset of 64 (fk_gelu.cuh);
// inputs below -30, -inf among them, give -0, the correctly rounded value.
// For bf16 outputs, where MUFU limits the kernel, the reciprocal is taken on
// the FMA pipes instead (a bit estimate and two Newton steps) and inputs are
// raised to -11, below which the result is -0 already.
//
// Exact form: x Phi(x), Phi the standard normal distribution function, with
// erfc in the form of Press et al. and coefficients fitted here (see
// fk_gelu.cuh).
//
// Errors stay within a few ulp of y: under 1e-6 absolute on [-20, 20] for
// fp32 (bound 2e-6), and within 1 ulp of the correctly rounded value for bf16.
#include "fk_common.cuh"
#include "fk_gelu.cuh"
#include "fk_internal.h"
#include "fk_sync.cuh"

namespace fk {

// Number of threads whose bounded mbarrier wait in the GELU / copy pipeline
// gave up (see fk_wait_timeouts).
__device__ unsigned int g_gelu_wait_timeouts = 0;

namespace {

constexpr size_t kMaxGrid = 0x7fffffffu;

struct CopyOp {
  __device__ __forceinline__ uint4 vec(uint4 v) const { return v; }
};

template <typename T, int KIND>
struct GeluOp {
  __device__ __forceinline__ uint4 vec(uint4 v) const {
    constexpr int VEC = Elem<T>::VEC;
    constexpr bool BF16 = sizeof(T) == 2;
    if constexpr (BF16) {  // clamped while packed
      v = make_uint4(max_nan_floor_bf16x2<KIND>(v.x), max_nan_floor_bf16x2<KIND>(v.y),
                     max_nan_floor_bf16x2<KIND>(v.z), max_nan_floor_bf16x2<KIND>(v.w));
    }
    float f[VEC];
    Elem<T>::unpack(v, f);
#pragma unroll
    for (int k = 0; k < VEC; k += 2) {
      const float2 g = gelu_f2<T, KIND, BF16>(make_float2(f[k], f[k + 1]));
      f[k] = g.x;
      f[k + 1] = g.y;
    }
    return Elem<T>::pack(f);
  }
};

// ---------------------------------------------------------------- through registers

// One block covers kRegThreads * kRegUnroll consecutive 16-byte vectors and
// each thread loads its kRegUnroll vectors before using any.  For working
// sets beyond L2 this grid streams at the copy rate, while grid-stride loops
// over a resident grid were 20% slower.
constexpr int kRegThreads = 256;
constexpr int kRegUnroll = 2;

template <typename Op>
__device__ __forceinline__ void stream_regs(const char* x, char* y, size_t nvec, Op op) {
  constexpr size_t kPerBlock = static_cast<size_t>(kRegThreads) * kRegUnroll;
  for (size_t b = blockIdx.x; b * kPerBlock < nvec; b += gridDim.x) {
    const size_t base = b * kPerBlock + threadIdx.x;
    uint4 v[kRegUnroll];
#pragma unroll
    for (int u = 0; u < kRegUnroll; ++u) {
      const size_t i = base + static_cast<size_t>(u) * kRegThreads;
      v[u] = ld_stream_v4_if(x + i * 16, i < nvec, 0u);
    }
#pragma unroll
    for (int u = 0; u < kRegUnroll; ++u) {
      const size_t i = base + static_cast<size_t>(u) * kRegThreads;
      st_stream_v4_if(y + i * 16, op.vec(v[u]), i < nvec);
    }
  }
}

size_t reg_blocks(size_t nvec) {
  const size_t per_block = static_cast<size_t>(kRegThreads) * kRegUnroll;
  const size_t b = (nvec + per_block - 1) / per_block;
  return b > kMaxGrid ? kMaxGrid : b;
}

// ---------------------------------------------------------------- through shared memory

// The vectors are cut into chunks of kChunkBytes.  Each block is persistent
// and walks the chunks blockIdx.x, blockIdx.x + gridDim.x, ...; it keeps
// kStages chunk loads in flight, each one cp.async.bulk (global -> shared)
// issued by one thread and completing on that stage's mbarrier.  When a
// stage lands, every thread takes its vectors from shared memory, computes
// in registers and stores them with 16-byte streaming stores (a warp's store
// covers 512 contiguous bytes); after a block barrier the stage is refilled
// with the block's chunk kStages further on.
constexpr uint32_t kChunkBytes = 16384;
constexpr int kStages = 3;
constexpr int kBulkBlocksPerSm = 4;
constexpr uint32_t kChunkVecs = kChunkBytes / 16;
constexpr size_t kStageSmem = static_cast<size_t>(kStages) * kChunkBytes;
constexpr uint64_t kBulkWaitNs = 1000000000ull;  // 1 s
// Threads per pipeline block, measured on B200 (32 MiB, mean of 60 launches,
// L2 cleaned / left dirty before each): fp32 streams best with 128 (tanh
// 12.3 / 14.3 us, exact 14.4 / 15.1); bf16, with twice the arithmetic per
// byte, with 256 (tanh 18.5 / 19.8 us against 18.5 / 20.4 with 128; exact
// 22.6 / 23.0 against 23.3 / 24.5).  512 was slower in every case.
constexpr int kCopyBulkThreads = 128;
template <typename T, int KIND>
struct GeluBulkThreads {
  static constexpr int value = sizeof(T) == 2 ? 256 : 128;
};

__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst_smem)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Bounded wait on a stage's mbarrier: false (and counted) after 1 s.
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kBulkWaitNs) {
      atomicAdd(&g_gelu_wait_timeouts, 1u);
      return false;
    }
  }
  return true;
}

// y = op(x) over `bytes` bytes (a multiple of 16) from 16-byte aligned x and
// y, chunk by chunk as described above, by blocks of THREADS threads.
template <int THREADS, typename Op>
__device__ __forceinline__ void stream_bulk(const char* x, char* y, size_t bytes, Op op) {
  static_assert(kChunkVecs % THREADS == 0, "whole vectors per thread in a chunk");
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int abort_flag;
  const int t = threadIdx.x;
  const size_t nchunks = (bytes + kChunkBytes - 1) / kChunkBytes;
  const size_t G = gridDim.x;
  const size_t nk = nchunks > blockIdx.x ? (nchunks - blockIdx.x + G - 1) / G : 0;
  if (nk == 0) return;  // the same for every thread of the block
  if (t == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  auto chunk_bytes = [&](size_t c) {
    const size_t off = c * kChunkBytes;
    return static_cast<uint32_t>(bytes - off < kChunkBytes ? bytes - off : kChunkBytes);
  };
  auto issue = [&](size_t k) {  // thread 0: the block's k-th chunk into stage k % kStages
    const size_t c = blockIdx.x + k * G;
    const int s = static_cast<int>(k % kStages);
    const uint32_t b = chunk_bytes(c);
    mbar_arrive_expect_tx(&full[s], b);
    bulk_load(stage_mem + s * kChunkBytes, x + c * kChunkBytes, b, &full[s]);
  };
  size_t issued = 0;
  if (t == 0) {
    for (; issued < nk && issued < static_cast<size_t>(kStages); ++issued) issue(issued);
  }
  size_t k = 0;
  for (; k < nk; ++k) {
    const int s = static_cast<int>(k % kStages);
    if (!stage_wait(&full[s], static_cast<uint32_t>((k / kStages) & 1))) abort_flag = 1;
    const size_t c = blockIdx.x + k * G;
    const uint32_t nv = chunk_bytes(c) / 16;
    const uint4* sv = reinterpret_cast<const uint4*>(stage_mem + s * kChunkBytes);
    uint4* yv = reinterpret_cast<uint4*>(y + c * kChunkBytes);
#pragma unroll
    for (int j = 0; j < static_cast<int>(kChunkVecs / THREADS); ++j) {
      const uint32_t vi = static_cast<uint32_t>(j * THREADS + t);
      if (vi < nv) st_stream_v4(yv + vi, op.vec(sv[vi]));
    }
    __syncthreads();  // every thread is done with stage s, and abort_flag is settled
    if (abort_flag) break;
    if (t == 0 && issued < nk) issue(issued++);
  }
  // After a wait that gave up, the loads still in flight land (bounded)
  // before the block exits: they write into its shared memory.
  if (abort_flag && t == 0) {
    for (size_t j = k; j < issued; ++j) stage_wait(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
  }
}

size_t bulk_blocks(size_t bytes, size_t scalar, int threads, int sm_count) {
  const size_t nchunks = (bytes + kChunkBytes - 1) / kChunkBytes;
  size_t blocks = static_cast<size_t>(sm_count > 0 ? sm_count : 1) * kBulkBlocksPerSm;
  if (blocks > nchunks) blocks = nchunks;
  const size_t scalar_blocks = (scalar + threads - 1) / threads;
  if (blocks < scalar_blocks) blocks = scalar_blocks;
  if (blocks > kMaxGrid) blocks = kMaxGrid;
  return blocks < 1 ? 1 : blocks;
}

// The stages and the static barriers exceed the 48 KB a block gets without
// opting in (set on every launch: the attribute is per device).
template <typename K>
cudaError_t allow_stage_smem(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kStageSmem));
}

// The shared-memory pipeline while input and output together fit in L2 and
// the input holds at least kBulkMinBytes: below that, one wave through
// registers has less fixed latency (measured alone with L2 cleaned, fp32
// tanh GELU: 1 MB 6.2 us against 8.1, 4 MB 6.6 against 8.1, 16 MB equal;
// the copy is equal either way up to 4 MB and faster through shared memory
// at 16 MB).
constexpr size_t kBulkMinBytes = size_t{8} << 20;
bool use_bulk(size_t bytes, size_t l2_bytes) { return bytes >= kBulkMinBytes && 2 * bytes <= l2_bytes; }

// ---------------------------------------------------------------- kernels

// x, y: the arrays.  Elements [0, head) and [tail_begin, n) are done with
// scalar accesses; [head, tail_begin) is nvec 16-byte vectors starting at a
// 16-byte boundary of both x and y.  BULK: through shared memory (above),
// by blocks of THREADS threads; otherwise through registers (kRegThreads).
template <typename T, int KIND, bool BULK, int THREADS>
__global__ void __launch_bounds__(THREADS)
    gelu_kernel(const T* x, T* y, size_t head, size_t nvec, size_t tail_begin, size_t n) {
  const size_t tid = static_cast<size_t>(blockIdx.x) * THREADS + threadIdx.x;
  const size_t nthr = static_cast<size_t>(gridDim.x) * THREADS;
  for (size_t i = tid; i < head; i += nthr) Elem<T>::store1(y + i, gelu_f<T, KIND>(Elem<T>::load1(x + i)));
  for (size_t i = tail_begin + tid; i < n; i += nthr)
    Elem<T>::store1(y + i, gelu_f<T, KIND>(Elem<T>::load1(x + i)));
  if constexpr (BULK) {
    stream_bulk<THREADS>(reinterpret_cast<const char*>(x + head), reinterpret_cast<char*>(y + head), nvec * 16,
                         GeluOp<T, KIND>{});
  } else {
    stream_regs(reinterpret_cast<const char*>(x + head), reinterpret_cast<char*>(y + head), nvec,
                GeluOp<T, KIND>{});
  }
}

// A plain copy through the same two paths: the achievable-bandwidth
// reference the fused kernels are measured against (fk_copy).
template <bool BULK>
__global__ void __launch_bounds__(BULK ? kCopyBulkThreads : kRegThreads)
    copy_kernel(const uint4* src, uint4* dst, size_t nvec) {
  if constexpr (BULK) {
    stream_bulk<kCopyBulkThreads>(reinterpret_cast<const char*>(src), reinterpret_cast<char*>(dst), nvec * 16,
                                  CopyOp{});
  } else {
    stream_regs(reinterpret_cast<const char*>(src), reinterpret_cast<char*>(dst), nvec, CopyOp{});
  }
}

template <typename T, int KIND>
cudaError_t launch_gelu_typed(const void* xp, void* yp, size_t n, const DeviceInfo& dev, cudaStream_t stream) {
  const T* x = static_cast<const T*>(xp);
  T* y = static_cast<T*>(yp);
  constexpr size_t VEC = Elem<T>::VEC;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
  size_t head = n, nvec = 0;
  if ((xa & 15) == (ya & 15)) {  // a common 16-byte phase: peel up to VEC-1 elements
    head = ((16 - (xa & 15)) & 15) / sizeof(T);
    if (head > n) head = n;
    nvec = (n - head) / VEC;
  }
  const size_t tail_begin = head + nvec * VEC;
  const size_t scalar = head > (n - tail_begin) ? head : (n - tail_begin);
  if (use_bulk(nvec * 16, dev.l2_bytes)) {
    constexpr int TB = GeluBulkThreads<T, KIND>::value;
    const cudaError_t e = allow_stage_smem(gelu_kernel<T, KIND, true, TB>);
    if (e != cudaSuccess) return e;
    gelu_kernel<T, KIND, true, TB><<<static_cast<unsigned>(bulk_blocks(nvec * 16, scalar, TB, dev.sm_count)), TB,
                                     kStageSmem, stream>>>(x, y, head, nvec, tail_begin, n);
  } else {
    size_t blocks = reg_blocks(nvec);
    const size_t scalar_blocks = (scalar + kRegThreads - 1) / kRegThreads;
    if (blocks < scalar_blocks) blocks = scalar_blocks;
    if (blocks < 1) blocks = 1;
    gelu_kernel<T, KIND, false, kRegThreads><<<static_cast<unsigned>(blocks), kRegThreads, 0, stream>>>(
        x, y, head, nvec, tail_begin, n);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gelu(const void* x, void* y, size_t n, int dtype, int kind, const DeviceInfo& dev,
                        cudaStream_t stream) {
  if (dtype == FK_F32) {
    return kind == FK_GELU_TANH ? launch_gelu_typed<float, FK_GELU_TANH>(x, y, n, dev, stream)
                                : launch_gelu_typed<float, FK_GELU_ERF>(x, y, n, dev, stream);
  }
  return kind == FK_GELU_TANH ? launch_gelu_typed<__nv_bfloat16, FK_GELU_TANH>(x, y, n, dev, stream)
                              : launch_gelu_typed<__nv_bfloat16, FK_GELU_ERF>(x, y, n, dev, stream);
}

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, const DeviceInfo& dev, cudaStream_t stream) {
  const size_t nvec = bytes / 16;
  if (nvec == 0) return cudaSuccess;
  const uint4* s = static_cast<const uint4*>(src);
  uint4* d = static_cast<uint4*>(dst);
  if (use_bulk(bytes, dev.l2_bytes)) {
    const cudaError_t e = allow_stage_smem(copy_kernel<true>);
    if (e != cudaSuccess) return e;
    copy_kernel<true><<<static_cast<unsigned>(bulk_blocks(bytes, 0, kCopyBulkThreads, dev.sm_count)),
                        kCopyBulkThreads, kStageSmem, stream>>>(s, d, nvec);
  } else {
    copy_kernel<false><<<static_cast<unsigned>(reg_blocks(nvec)), kRegThreads, 0, stream>>>(s, d, nvec);
  }
  return cudaGetLastError();
}

cudaError_t read_gelu_wait_timeouts(unsigned* out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_gelu_wait_timeouts, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_gelu_wait_timeouts, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace fk
