// fk_api.cu -- the C ABI of libfk (declared in include/fk.h): argument
// validation, the per-device properties cache, and dispatch to the kernels.
//
// Every check runs on the host before anything is enqueued, so a rejected
// call launches nothing.  Pointer checks use the CUDA runtime's pointer
// attributes (pageable host memory is not device-accessible) and the
// driver's address-range query (the whole [ptr, ptr + bytes) span must lie
// inside one allocation), which turns a wrong size into an error code
// instead of a device fault.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cfloat>

#include <stdint.h>

#include <atomic>
#include <mutex>

#include "fk.h"
#include "fk_internal.h"

namespace fk {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kVersion = 10000;  // 1.0.0

DeviceInfo g_info[kMaxDevices];
std::once_flag g_info_once[kMaxDevices];
thread_local int t_last_cuda_error = 0;

// Private stream-ordered memory pool per device for the split path's
// workspace.  Its release threshold keeps up to 64 MiB reserved across
// synchronisations, so repeated calls reuse memory instead of going back to
// the driver (the default pool's threshold of 0 made every call a fresh
// allocation).  A private pool leaves the process-wide default pool as it is.
std::once_flag g_pool_once[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices] = {};

cudaMemPool_t workspace_pool(int dev) {
  std::call_once(g_pool_once[dev], [dev] {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
      (void)cudaGetLastError();
      return;
    }
    uint64_t keep = uint64_t{64} << 20;
    (void)cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pool[dev] = pool;
  });
  return g_pool[dev];
}

}  // namespace

// Stream-ordered workspace from the private pool of the current device (the
// default pool if the private one could not be made).
cudaError_t workspace_alloc(void** p, size_t bytes, cudaStream_t s) {
  int d = -1;
  const cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return e;
  const cudaMemPool_t pool = (d >= 0 && d < kMaxDevices) ? workspace_pool(d) : nullptr;
  return pool ? cudaMallocFromPoolAsync(p, bytes, pool, s) : cudaMallocAsync(p, bytes, s);
}

namespace {

fk_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FK_ERR_CUDA;
}

void query_device(int dev) {
  DeviceInfo& d = g_info[dev];
  d.ok = 0;
  cudaDeviceProp p;
  if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return;
  d.major = p.major;
  d.minor = p.minor;
  d.sm_count = p.multiProcessorCount;
  d.max_threads_sm = p.maxThreadsPerMultiProcessor;
  d.l2_bytes = static_cast<size_t>(p.l2CacheSize);
  d.ok = 1;
}

// cuMemGetAddressRange, resolved once through the runtime so that libfk
// needs no link-time dependency on the driver library.
typedef CUresult (*PFN_addr_range)(CUdeviceptr*, size_t*, CUdeviceptr);
std::atomic<PFN_addr_range> g_addr_range{nullptr};
std::once_flag g_addr_range_once;

PFN_addr_range addr_range_fn() {
  std::call_once(g_addr_range_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_addr_range.store(reinterpret_cast<PFN_addr_range>(fn));
  });
  return g_addr_range.load();
}

// Is [p, p + bytes) memory the current device `dev` may access?
fk_status check_pointer(const void* p, size_t bytes, int dev) {
  cudaPointerAttributes a;
  const cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // clear the non-sticky error
    return FK_ERR_INVALID_ARG;
  }
  switch (a.type) {
    case cudaMemoryTypeDevice:
      if (a.device != dev) return FK_ERR_INVALID_ARG;
      break;
    case cudaMemoryTypeManaged:
      break;
    case cudaMemoryTypeHost:
      if (a.devicePointer == nullptr) return FK_ERR_INVALID_ARG;
      break;
    default:  // unregistered (pageable) host memory
      return FK_ERR_INVALID_ARG;
  }
  if (a.type == cudaMemoryTypeDevice) {
    if (PFN_addr_range f = addr_range_fn()) {
      CUdeviceptr base = 0;
      size_t size = 0;
      // device memory whose extent cannot be established is not accepted
      if (f(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return FK_ERR_INVALID_ARG;
      const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
      if (lo < base || lo - base > size || bytes > size - (lo - base)) return FK_ERR_INVALID_ARG;
    }
  }
  return FK_OK;
}

bool overlaps_partially(const void* x, const void* y, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
  if (a == b) return false;  // exact aliasing: in place, allowed
  return a < b + bytes && b < a + bytes;
}

// Common checks for one (x, y, element count, element size) call.
fk_status check_call(const void* x, const void* y, size_t count, size_t esize,
                     const DeviceInfo** dev_out) {
  if (x == nullptr || y == nullptr) return FK_ERR_INVALID_ARG;
  if (count > SIZE_MAX / esize) return FK_ERR_INVALID_ARG;
  const size_t bytes = count * esize;
  if ((reinterpret_cast<uintptr_t>(x) % esize) != 0 || (reinterpret_cast<uintptr_t>(y) % esize) != 0)
    return FK_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) > UINTPTR_MAX - bytes ||
      reinterpret_cast<uintptr_t>(y) > UINTPTR_MAX - bytes)
    return FK_ERR_INVALID_ARG;
  if (overlaps_partially(x, y, bytes)) return FK_ERR_INVALID_ARG;
  int dev = -1;
  const DeviceInfo* info = current_device_info(&dev);
  if (info == nullptr || !info->ok) return FK_ERR_UNSUPPORTED_DEVICE;
  if (info->major != 10 || info->minor != 0) return FK_ERR_UNSUPPORTED_DEVICE;
  fk_status st = check_pointer(x, bytes, dev);
  if (st != FK_OK) return st;
  if (y != x) {
    st = check_pointer(y, bytes, dev);
    if (st != FK_OK) return st;
  }
  *dev_out = info;
  return FK_OK;
}

}  // namespace

fk_status validate_call(const void* x, const void* y, size_t count, size_t esize) {
  const DeviceInfo* dev = nullptr;
  return check_call(x, y, count, esize, &dev);
}

const DeviceInfo* current_device_info(int* device_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_info_once[dev], query_device, dev);
  if (device_out) *device_out = dev;
  return &g_info[dev];
}

}  // namespace fk

extern "C" {

fk_status fk_gelu(const void* x, void* y, size_t n, int dtype, int kind, void* stream) {
  if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED_DTYPE;
  if (kind != FK_GELU_TANH && kind != FK_GELU_ERF) return FK_ERR_INVALID_ARG;
  if (n == 0) return FK_OK;
  const fk::DeviceInfo* dev = nullptr;
  const fk_status st = fk::check_call(x, y, n, dtype == FK_F32 ? 4 : 2, &dev);
  if (st != FK_OK) return st;
  const cudaError_t e = fk::launch_gelu(x, y, n, dtype, kind, *dev, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

fk_status fk_copy(const void* src, void* dst, size_t bytes, void* stream) {
  if (bytes == 0) return FK_OK;
  if (bytes % 16 != 0 || reinterpret_cast<uintptr_t>(src) % 16 != 0 || reinterpret_cast<uintptr_t>(dst) % 16 != 0)
    return FK_ERR_INVALID_ARG;
  if (src == dst) return FK_ERR_INVALID_ARG;
  const fk::DeviceInfo* dev = nullptr;
  const fk_status st = fk::check_call(src, dst, bytes / 16, 16, &dev);
  if (st != FK_OK) return st;
  const cudaError_t e = fk::launch_copy(src, dst, bytes, *dev, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

fk_status fk_gelu_tanh(const float* x, float* y, size_t n, void* stream) {
  return fk_gelu(x, y, n, FK_F32, FK_GELU_TANH, stream);
}

fk_status fk_softmax_rows_plan(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out) {
  return fk::plan_softmax(rows, cols, dtype, path, out);
}

namespace {

// Resolve the plan of a softmax call (auto or explicit).
fk_status resolve_plan(size_t rows, size_t cols, int dtype, const fk_softmax_plan* plan, fk_softmax_plan* p) {
  if (plan == nullptr || plan->path == FK_PATH_AUTO) return fk::plan_softmax(rows, cols, dtype, FK_PATH_AUTO, p);
  return fk::check_plan(rows, cols, dtype, *plan, p);
}

// Shared body of the softmax entry points.  ws == nullptr and
// allow_alloc: a needed workspace is allocated stream-ordered.
// sc == nullptr: plain softmax.
fk_status softmax_call(const void* x, void* y, size_t rows, size_t cols, int dtype, const fk_softmax_plan* plan,
                       void* ws, size_t ws_bytes, bool allow_alloc, const fk::SoftmaxScaling* sc, void* stream) {
  if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED_DTYPE;
  if (rows == 0 || cols == 0) return FK_OK;
  if (rows > SIZE_MAX / cols) return FK_ERR_INVALID_ARG;
  fk_softmax_plan p;
  fk_status st = resolve_plan(rows, cols, dtype, plan, &p);
  if (st != FK_OK) return st;
  const size_t esize = dtype == FK_F32 ? 4 : 2;
  const fk::DeviceInfo* dev = nullptr;
  st = fk::check_call(x, y, rows * cols, esize, &dev);
  if (st != FK_OK) return st;
  const size_t need = fk::workspace_bytes(rows, cols, dtype, p);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool owned = false;
  if (need > 0) {
    if (ws != nullptr) {
      if (ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) % 8) != 0) return FK_ERR_INVALID_ARG;
      const size_t data = rows * cols * esize;
      const uintptr_t w = reinterpret_cast<uintptr_t>(ws);
      const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
      if ((w < a + data && a < w + need) || (w < b + data && b < w + need)) return FK_ERR_INVALID_ARG;
      int d = -1;
      if (cudaGetDevice(&d) != cudaSuccess) return FK_ERR_UNSUPPORTED_DEVICE;
      st = fk::check_pointer(ws, need, d);
      if (st != FK_OK) return st;
    } else {
      if (!allow_alloc) return FK_ERR_INVALID_ARG;
      int d = -1;
      if (cudaGetDevice(&d) != cudaSuccess) return FK_ERR_UNSUPPORTED_DEVICE;
      const cudaMemPool_t pool = fk::workspace_pool(d);
      const cudaError_t e = pool ? cudaMallocFromPoolAsync(&ws, need, pool, s) : cudaMallocAsync(&ws, need, s);
      if (e != cudaSuccess) return fk::cuda_fail(e);
      owned = true;
    }
  }
  // 16-byte vector access needs both bases on a 16-byte boundary and a row
  // pitch that is a multiple of 16 bytes.
  const bool aligned = (reinterpret_cast<uintptr_t>(x) % 16 == 0) &&
                       (reinterpret_cast<uintptr_t>(y) % 16 == 0) && ((cols * esize) % 16 == 0);
  cudaError_t e = fk::launch_softmax(x, y, rows, cols, dtype, p, aligned, ws, sc, *dev, s);
  if (owned) {
    const cudaError_t f = cudaFreeAsync(ws, s);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

}  // namespace

fk_status fk_softmax_rows_ex(const void* x, void* y, size_t rows, size_t cols, int dtype,
                             const fk_softmax_plan* plan, void* stream) {
  return softmax_call(x, y, rows, cols, dtype, plan, nullptr, 0, true, nullptr, stream);
}

fk_status fk_softmax_rows_ws(const void* x, void* y, size_t rows, size_t cols, int dtype,
                             const fk_softmax_plan* plan, void* workspace, size_t workspace_bytes, void* stream) {
  return softmax_call(x, y, rows, cols, dtype, plan, workspace, workspace_bytes, false, nullptr, stream);
}

fk_status fk_softmax_rows_causal_ex(const void* x, void* y, size_t rows, size_t cols, int dtype, float scale,
                                    size_t period, size_t offset, unsigned int flags, const fk_softmax_plan* plan,
                                    void* stream) {
  if (!(scale > 0.0f) || !(scale <= FLT_MAX)) return FK_ERR_INVALID_ARG;  // also rejects NaN
  if ((flags & ~FK_SOFTMAX_SKIP_MASKED) != 0) return FK_ERR_INVALID_ARG;
  fk::SoftmaxScaling sc;
  sc.k = static_cast<float>(static_cast<double>(scale) * 1.44269504088896340736);
  // (r mod period) + offset: a period beyond the rows and an offset beyond
  // the columns change nothing, and bounding them keeps the sum from wrapping
  sc.period = period < rows ? period : rows;
  sc.offset = offset < cols ? offset : cols;
  sc.row0 = 0;
  sc.skip_masked = (flags & FK_SOFTMAX_SKIP_MASKED) ? 1 : 0;
  fk::set_period_division(&sc, rows);
  return softmax_call(x, y, rows, cols, dtype, plan, nullptr, 0, true, &sc, stream);
}

fk_status fk_layernorm_rows_ex(const void* x, void* y, const float* gamma, const float* beta, size_t rows,
                               size_t cols, int dtype, float eps, int epilogue, const fk_softmax_plan* plan,
                               void* stream) {
  if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED_DTYPE;
  if (!(eps >= 0.0f) || !(eps <= FLT_MAX)) return FK_ERR_INVALID_ARG;
  if (epilogue != FK_EPILOGUE_NONE && epilogue != FK_EPILOGUE_GELU_TANH && epilogue != FK_EPILOGUE_GELU_ERF)
    return FK_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return FK_OK;
  if (rows > SIZE_MAX / cols) return FK_ERR_INVALID_ARG;
  fk_softmax_plan p;
  fk_status st = (plan == nullptr || plan->path == FK_PATH_AUTO)
                     ? fk::plan_layernorm(rows, cols, dtype, FK_PATH_AUTO, &p)
                     : fk::check_layernorm_plan(rows, cols, dtype, *plan, &p);
  if (st != FK_OK) return st;
  const size_t esize = dtype == FK_F32 ? 4 : 2;
  const fk::DeviceInfo* dev = nullptr;
  st = fk::check_call(x, y, rows * cols, esize, &dev);
  if (st != FK_OK) return st;
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) return FK_ERR_UNSUPPORTED_DEVICE;
  const size_t pbytes = cols * sizeof(float);
  const uintptr_t yb = reinterpret_cast<uintptr_t>(y);
  const size_t ybytes = rows * cols * esize;
  for (const float* q : {gamma, beta}) {
    if (q == nullptr) continue;
    const uintptr_t a = reinterpret_cast<uintptr_t>(q);
    if (a % sizeof(float) != 0 || a > UINTPTR_MAX - pbytes) return FK_ERR_INVALID_ARG;
    if (a < yb + ybytes && yb < a + pbytes) return FK_ERR_INVALID_ARG;  // the output would overwrite it
    st = fk::check_pointer(q, pbytes, d);
    if (st != FK_OK) return st;
  }
  const bool aligned = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (yb % 16 == 0) &&
                       ((cols * esize) % 16 == 0) && (reinterpret_cast<uintptr_t>(gamma) % 16 == 0) &&
                       (reinterpret_cast<uintptr_t>(beta) % 16 == 0);
  const cudaError_t e = fk::launch_layernorm(x, y, gamma, beta, rows, cols, dtype, eps, epilogue, p, aligned,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

fk_status fk_layernorm_rows_plan(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out) {
  return fk::plan_layernorm(rows, cols, dtype, path, out);
}

fk_status fk_layernorm_rows(const void* x, void* y, const float* gamma, const float* beta, size_t rows,
                            size_t cols, int dtype, float eps, int epilogue, void* stream) {
  return fk_layernorm_rows_ex(x, y, gamma, beta, rows, cols, dtype, eps, epilogue, nullptr, stream);
}

fk_status fk_softmax_rows_causal(const void* x, void* y, size_t rows, size_t cols, int dtype, float scale,
                                 size_t period, size_t offset, void* stream) {
  return fk_softmax_rows_causal_ex(x, y, rows, cols, dtype, scale, period, offset, 0, nullptr, stream);
}

fk_status fk_softmax_rows_workspace(size_t rows, size_t cols, int dtype, const fk_softmax_plan* plan,
                                    size_t* bytes) {
  if (bytes == nullptr) return FK_ERR_INVALID_ARG;
  if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED_DTYPE;
  if (rows == 0 || cols == 0) {
    *bytes = 0;
    return FK_OK;
  }
  fk_softmax_plan p;
  const fk_status st = resolve_plan(rows, cols, dtype, plan, &p);
  if (st != FK_OK) return st;
  *bytes = fk::workspace_bytes(rows, cols, dtype, p);
  return FK_OK;
}

fk_status fk_softmax_rows(const void* x, void* y, size_t rows, size_t cols, int dtype, void* stream) {
  return fk_softmax_rows_ex(x, y, rows, cols, dtype, nullptr, stream);
}

fk_status fk_wait_timeouts(unsigned int* count, int reset) {
  if (count == nullptr) return FK_ERR_INVALID_ARG;
  int dev = -1;
  const fk::DeviceInfo* info = fk::current_device_info(&dev);
  if (info == nullptr || !info->ok) return FK_ERR_UNSUPPORTED_DEVICE;
  if (info->major != 10 || info->minor != 0) return FK_ERR_UNSUPPORTED_DEVICE;
  unsigned a = 0, b = 0, c = 0;
  cudaError_t e = fk::read_wait_timeouts(&a, reset != 0);
  if (e == cudaSuccess) e = fk::read_attention_wait_timeouts(&b, reset != 0);
  if (e == cudaSuccess) e = fk::read_gelu_wait_timeouts(&c, reset != 0);
  *count = a + b + c;
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

fk_status fk_attention_fwd(const void* q, const void* k, const void* v, void* o, size_t bh, size_t t, size_t d,
                           int causal, float scale, void* stream) {
  if (causal != 0 && causal != 1) return FK_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !(scale <= FLT_MAX)) return FK_ERR_INVALID_ARG;
  if (bh == 0 || t == 0) return FK_OK;
  if ((d != 64 && d != 128) || t % 128 != 0 || t / 128 > 65535) return FK_ERR_INVALID_ARG;
  if (bh > (size_t{1} << 31) / t || bh * t >= (size_t{1} << 31)) return FK_ERR_INVALID_ARG;
  const size_t n = bh * t * d;
  const size_t bytes = n * 2;
  for (const void* p : {q, k, v, static_cast<const void*>(o)})
    if (p == nullptr || reinterpret_cast<uintptr_t>(p) % 16 != 0) return FK_ERR_INVALID_ARG;
  const uintptr_t ob = reinterpret_cast<uintptr_t>(o);
  for (const void* p : {q, k, v}) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (a < ob + bytes && ob < a + bytes) return FK_ERR_INVALID_ARG;  // the output may not overlap an input
  }
  const fk::DeviceInfo* dev = nullptr;
  fk_status st = fk::check_call(q, o, n, 2, &dev);
  if (st != FK_OK) return st;
  int di = -1;
  if (cudaGetDevice(&di) != cudaSuccess) return FK_ERR_UNSUPPORTED_DEVICE;
  for (const void* p : {k, v}) {
    st = fk::check_pointer(p, bytes, di);
    if (st != FK_OK) return st;
  }
  const cudaError_t e = fk::launch_attention(q, k, v, o, bh, t, static_cast<int>(d), causal != 0, scale,
                                             dev->sm_count, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

fk_status fk_wait_selftest(unsigned int timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 10000000u) return FK_ERR_INVALID_ARG;
  int dev = -1;
  const fk::DeviceInfo* info = fk::current_device_info(&dev);
  if (info == nullptr || !info->ok) return FK_ERR_UNSUPPORTED_DEVICE;
  if (info->major != 10 || info->minor != 0) return FK_ERR_UNSUPPORTED_DEVICE;
  const cudaError_t e = fk::launch_wait_selftest(timeout_us, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FK_OK : fk::cuda_fail(e);
}

const char* fk_status_string(int status) {
  switch (status) {
    case FK_OK: return "FK_OK: success";
    case FK_ERR_INVALID_ARG: return "FK_ERR_INVALID_ARG: invalid argument (pointer, size, alignment, overlap or plan)";
    case FK_ERR_UNSUPPORTED_DTYPE: return "FK_ERR_UNSUPPORTED_DTYPE: dtype must be FK_F32 or FK_BF16";
    case FK_ERR_UNSUPPORTED_DEVICE: return "FK_ERR_UNSUPPORTED_DEVICE: no CUDA device, or not sm_100 (B200)";
    case FK_ERR_CUDA: return "FK_ERR_CUDA: a CUDA call or kernel launch failed (see fk_last_cuda_error)";
    default: return "unknown fk_status";
  }
}

int fk_last_cuda_error(void) { return fk::t_last_cuda_error; }

int fk_version(void) { return fk::kVersion; }

}  // extern "C"
