// fk_noalloc.cu -- fk_softmax_rows_noalloc: row softmax that never allocates
// device memory, for callers that cannot call cudaMalloc (or have the library
// do so): code running under a framework that has reserved nearly all device
// memory for its own allocator, latency-critical loops that cannot afford an
// allocation call (cudaMalloc may synchronise the device), and environments
// whose policy forbids a library from allocating.
//
// Only the split path (few or very long rows) needs scratch memory: one
// (max, sum) pair per chunk of the rows of a launch.  Here that scratch is a
// file-scope device array of fixed size, part of the library image: every
// GPU that loads the library holds it (1 MiB) until the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fk.h"
#include "fk_internal.h"

namespace fk {
namespace {

constexpr size_t kNoAllocPartials = 131072;  // float2 pairs: 1 MiB
static_assert(kNoAllocPartials * sizeof(float2) == (size_t{1} << 20), "1 MiB of scratch");

// The scratch of every fk_softmax_rows_noalloc call on a device.  Shared by
// all calls; it keeps the contents of the last call.  Nothing in it needs to
// start at zero: a call's stats kernel writes every partial that its
// normalise kernel reads, before that kernel runs.
static __device__ __align__(256) float2 g_noalloc_scratch[kNoAllocPartials];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on device `dev`, which must be the
// current device.  (In host code the array's name is only a host-side
// stand-in; a kernel given it would read the wrong memory or fault.)
// A successful lookup is kept for the life of the process; a failed one
// (for example inside a stream capture) is not, and the next call retries.
void* scratch_address(int dev, cudaError_t* err) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  *err = cudaSuccess;
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      *err = e;
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace fk

namespace fk {
namespace {

// The allocation-free call with a scratch of `capacity` (max, sum) pairs
// (at most the array's).  Rows run in batches of floor(capacity / chunks)
// rows, chunks as planned for all rows; each batch plans its own chunking
// for its row count, so the two batch sizes that occur (the full batch and
// the shorter last one) are checked against the capacity before anything
// is enqueued.
fk_status noalloc_batched(const void* x, void* y, size_t rows, size_t cols, int dtype, size_t capacity,
                          void* stream) {
  if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED_DTYPE;
  if (rows == 0 || cols == 0) return FK_OK;
  if (rows > SIZE_MAX / cols) return FK_ERR_INVALID_ARG;
  fk_softmax_plan plan;
  fk_status st = plan_softmax(rows, cols, dtype, FK_PATH_AUTO, &plan);
  if (st != FK_OK) return st;
  if (plan.path != FK_PATH_SPLIT) {
    // every other path keeps its state on chip: nothing to allocate
    return fk_softmax_rows_ws(x, y, rows, cols, dtype, &plan, nullptr, 0, stream);
  }
  // A single row with more chunks than the scratch holds (for the whole
  // array: more than 2^35 elements) is refused.  The whole of x and y is
  // checked before the first batch is enqueued, so a rejected call writes
  // nothing.
  const SplitGeometry g = split_geometry(rows, cols, dtype);
  if (g.nchunks > capacity) return FK_ERR_INVALID_ARG;
  const size_t rows_per_batch = capacity / g.nchunks;
  const size_t last = rows % rows_per_batch;
  const size_t cap_bytes = capacity * sizeof(float2);
  if (split_geometry(rows < rows_per_batch ? rows : rows_per_batch, cols, dtype).ws_bytes > cap_bytes ||
      (last != 0 && split_geometry(last, cols, dtype).ws_bytes > cap_bytes))
    return FK_ERR_INVALID_ARG;
  const size_t esize = dtype == FK_F32 ? 4 : 2;
  st = validate_call(x, y, rows * cols, esize);
  if (st != FK_OK) return st;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return FK_ERR_UNSUPPORTED_DEVICE;
  }
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(dev, &err);
  if (scratch == nullptr) return FK_ERR_CUDA;
  const char* xb = static_cast<const char*>(x);
  char* yb = static_cast<char*>(y);
  for (size_t r0 = 0; r0 < rows; r0 += rows_per_batch) {
    const size_t n = (rows - r0 < rows_per_batch) ? rows - r0 : rows_per_batch;
    fk_softmax_plan p = plan;
    p.chunks = 0;
    const size_t off = r0 * cols * esize;
    st = fk_softmax_rows_ws(xb + off, yb + off, n, cols, dtype, &p, scratch, cap_bytes, stream);
    if (st != FK_OK) return st;
  }
  return FK_OK;
}

}  // namespace
}  // namespace fk

extern "C" fk_status fk_softmax_rows_noalloc(const void* x, void* y, size_t rows, size_t cols, int dtype,
                                             void* stream) {
  return fk::noalloc_batched(x, y, rows, cols, dtype, fk::kNoAllocPartials, stream);
}

extern "C" fk_status fk_softmax_rows_noalloc_cap(const void* x, void* y, size_t rows, size_t cols, int dtype,
                                                 size_t capacity_pairs, void* stream) {
  if (capacity_pairs == 0 || capacity_pairs > fk::kNoAllocPartials) return FK_ERR_INVALID_ARG;
  return fk::noalloc_batched(x, y, rows, cols, dtype, capacity_pairs, stream);
}
