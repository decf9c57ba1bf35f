// fk_internal.h -- host-side interfaces between the C ABI (fk_api.cu) and the
// kernel launchers (fk_gelu.cu, fk_softmax.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fk.h"

namespace fk {

// Cached properties of one device (filled once per device id).
struct DeviceInfo {
  int ok;               // 1 if the query succeeded
  int major, minor;     // compute capability
  int sm_count;         // multiprocessors
  int max_threads_sm;   // resident threads per multiprocessor
  size_t l2_bytes;      // L2 cache size
};

// Properties of the current device; nullptr if there is none.
const DeviceInfo* current_device_info(int* device_out);

// The checks every (x, y) entry point runs for `count` elements of `esize`
// bytes: non-null, element-aligned, no partial overlap, an sm_100 current
// device, and both spans inside device-accessible allocations.
fk_status validate_call(const void* x, const void* y, size_t count, size_t esize);

// ---- GELU --------------------------------------------------------------
// y[i] = GELU(x[i]) for i < n, dtype FK_F32 / FK_BF16, kind FK_GELU_TANH /
// FK_GELU_ERF.  Arguments already validated; the device's L2 size and SM
// count choose the path and size the grid.
cudaError_t launch_gelu(const void* x, void* y, size_t n, int dtype, int kind, const DeviceInfo& dev,
                        cudaStream_t stream);

// dst <- src, bytes a multiple of 16 and both 16-byte aligned (validated).
cudaError_t launch_copy(const void* src, void* dst, size_t bytes, const DeviceInfo& dev, cudaStream_t stream);

// Threads whose bounded wait in the GELU / copy kernels gave up (see
// read_wait_timeouts).
cudaError_t read_gelu_wait_timeouts(unsigned* out, bool reset);

// ---- softmax -----------------------------------------------------------
constexpr int kWarpRowsPerBlock = 8;        // warps (= rows) per block on the warp path, at most
constexpr int kWarpThreads = 32 * kWarpRowsPerBlock;
constexpr int kBlockEptSmall = 16;          // register-resident elements per thread (CTA/cluster)
constexpr int kBlockEptLarge = 32;
constexpr int kClusterEpt = 64;             // cluster blocks: 64 values per thread, <= 512 threads
constexpr int kTwoPhaseThreads = 512;
constexpr int kTwoPhaseElemsPerThread = 16; // elements per thread per streamed chunk
constexpr int kMaxCluster = 16;

// Vectors (16 bytes) per thread implied by a dtype and an element budget.
int vec_elems(int dtype);  // 4 for fp32, 8 for bf16

// Geometry of the split path (FK_PATH_SPLIT): each row is cut into nchunks
// chunks of chunk_vecs 16-byte vectors, one block per chunk; rows go in
// batches of rows_per_launch, whose partials fit ws_bytes of workspace.
struct SplitGeometry {
  size_t chunk_vecs;
  unsigned nchunks;
  size_t rows_per_launch;
  size_t ws_bytes;
};
SplitGeometry split_geometry(size_t rows, size_t cols, int dtype);

// Host-only plan (see fk_softmax_rows_plan in fk.h).
fk_status plan_softmax(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out);
// Validate a caller-provided plan and fill defaults.
fk_status check_plan(size_t rows, size_t cols, int dtype, const fk_softmax_plan& in, fk_softmax_plan* out);

// Scale and causal mask of fk_softmax_rows_causal.  Row r (counted from the
// start of the whole call) keeps columns j < limit(r), limit(r) =
// min(cols, (r mod period) + offset + 1), or every column when period == 0,
// and computes softmax(scale * x_j) over them; the other columns are not
// read and are written 0 (or, with skip_masked, not written where a whole
// 16-byte vector is masked).
struct SoftmaxScaling {
  float k;        // scale * log2(e), rounded once to fp32
  size_t period;  // 0: no mask; otherwise 1 <= period <= rows
  size_t offset;  // <= cols
  size_t row0;    // index of the launch's first row within the call (set by the launchers)
  // r mod period by multiplication (Granlund and Montgomery, "Division by
  // invariant integers using multiplication", 1994, unsigned 32-bit case):
  // q = (t + ((n - t) >> shift1)) >> shift2 with t = mulhi(magic, n).  Used
  // when fast32 is set (period and every row index below 2^32).
  uint32_t magic, shift1, shift2;
  int fast32;
  int skip_masked;  // 1: masked columns are not stored (FK_SOFTMAX_SKIP_MASKED)
};

// Fill the division fields of `sc` for its period and the call's rows.
void set_period_division(SoftmaxScaling* sc, size_t rows);

// Launch a validated plan.  `aligned` = rows and both pointers allow 16-byte
// vector access.
// `ws` is device workspace of at least workspace_bytes(plan) bytes (only the
// split path uses it; may be null otherwise).  `sc` == nullptr: plain
// softmax; otherwise scaled and masked as above.
cudaError_t launch_softmax(const void* x, void* y, size_t rows, size_t cols, int dtype,
                           const fk_softmax_plan& plan, bool aligned, void* ws, const SoftmaxScaling* sc,
                           const DeviceInfo& dev, cudaStream_t stream);

// ---- LayerNorm -----------------------------------------------------------
// Plan of fk_layernorm_rows: FK_PATH_WARP (cols <= 1024 fp32 / 2048 bf16 on
// demand), FK_PATH_CTA (<= 32768) or FK_PATH_TWOPHASE (any length: one
// 512-thread block per row streams it twice).  `path` = FK_PATH_AUTO or one
// of those; a caller plan is validated by check_layernorm_plan.
fk_status plan_layernorm(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out);
fk_status check_layernorm_plan(size_t rows, size_t cols, int dtype, const fk_softmax_plan& in,
                               fk_softmax_plan* out);

// Launch a validated LayerNorm plan (gamma / beta: fp32 device arrays of
// cols values, or nullptr; `aligned`: x, y, gamma and beta allow 16-byte
// vector access along rows).
cudaError_t launch_layernorm(const void* x, void* y, const float* gamma, const float* beta, size_t rows,
                             size_t cols, int dtype, float eps, int epilogue, const fk_softmax_plan& plan,
                             bool aligned, cudaStream_t stream);

// Workspace bytes a validated plan needs (0 except on the split path).
size_t workspace_bytes(size_t rows, size_t cols, int dtype, const fk_softmax_plan& plan);

// Stream-ordered device workspace of `bytes` from the library's private pool
// on the current device (kept reserved across calls); release it with
// cudaFreeAsync on the same stream after the kernels that use it.
cudaError_t workspace_alloc(void** p, size_t bytes, cudaStream_t s);

// ---- attention ------------------------------------------------------------
// O = softmax(scale Q K^T, causal) V over bh slices of [t, d] bf16 rows
// (validated: t % 128 == 0, d in {64, 128}, 16-byte aligned, bh * t < 2^31).
cudaError_t launch_attention(const void* q, const void* k, const void* v, void* o, size_t bh, size_t t, int d,
                             bool causal, float scale, int sm_count, cudaStream_t stream);
cudaError_t read_attention_wait_timeouts(unsigned* out, bool reset);

// Number of threads whose bounded mbarrier wait gave up, on the current
// device; optionally reset to 0.  Synchronous.
cudaError_t read_wait_timeouts(unsigned* out, bool reset);

// One block of 32 threads waits on an mbarrier that nothing arrives on and
// gives up after timeout_us microseconds (adds 32 to the count above).
cudaError_t launch_wait_selftest(unsigned timeout_us, cudaStream_t stream);

}  // namespace fk
