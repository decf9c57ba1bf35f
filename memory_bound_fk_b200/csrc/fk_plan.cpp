// fk_plan.cpp -- host-only choice of the softmax kernel for a row length.
//
// The capacities follow from the kernels' register budgets:
//   warp     : 32 lanes x VPT 16-byte vectors, VPT in {1, 2, 4, 8}
//              -> up to 1024 fp32 / 2048 bf16 columns
//   block    : 16 or 32 elements per thread (EPT), threads in
//              {128, 256, 512, 1024} -> up to 32768 columns
//   cluster  : 2..16 blocks of 128..512 threads holding 64 values each
//              -> up to 524288 columns
//   twophase : any length (row streamed twice)
// The automatic choice takes the smallest shape that holds the row on chip,
// so a row is read from HBM once whenever it fits in a cluster.  Measured on
// B200 (L2 cleaned between runs): 4096-column fp32 rows run best as one
// 128-thread block with 32 elements per thread; 2048-column bf16 rows as one
// 128-thread block with 16 elements per thread (32 registers, so 16 blocks
// fit per SM); rows up to 1024 fp32 / bf16 columns stay on one warp;
// 131072-column fp32 rows as a cluster of 16 blocks of 128 threads with 64
// values per thread (more, smaller blocks fit more clusters on the GPU).
#include <stddef.h>

#include "fk_internal.h"

namespace fk {

int vec_elems(int dtype) { return dtype == FK_BF16 ? 8 : 4; }

namespace {

bool valid_dtype(int dtype) { return dtype == FK_F32 || dtype == FK_BF16; }

size_t ceil_div(size_t a, size_t b) { return (a + b - 1) / b; }

bool block_threads_ok(int t) { return t == 128 || t == 256 || t == 512 || t == 1024; }

size_t warp_cap(int dtype, int vpt) { return static_cast<size_t>(32) * vpt * vec_elems(dtype); }

size_t block_cap(int threads, int ept) { return static_cast<size_t>(threads) * ept; }

bool ept_ok(int ept) { return ept == kBlockEptSmall || ept == kBlockEptLarge; }

bool cluster_ept_ok(int ept, int threads) {
  return ept_ok(ept) || (ept == kClusterEpt && threads <= 512);
}

}  // namespace

fk_status plan_softmax(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out) {
  (void)rows;
  if (!valid_dtype(dtype)) return FK_ERR_UNSUPPORTED_DTYPE;
  if (out == nullptr || cols == 0) return FK_ERR_INVALID_ARG;
  const int vec = vec_elems(dtype);
  // elements per thread on the block paths: bf16 rows use the small budget
  // while it suffices (fewer registers, more resident blocks)
  const int ept_cta = (dtype == FK_BF16 && cols <= block_cap(1024, kBlockEptSmall)) ? kBlockEptSmall
                                                                                    : kBlockEptLarge;
  if (path == FK_PATH_AUTO) {
    if (cols <= 1024)
      path = FK_PATH_WARP;
    else if (cols <= block_cap(1024, kBlockEptLarge))
      path = FK_PATH_CTA;
    else if (cols <= static_cast<size_t>(kMaxCluster) * block_cap(1024, kBlockEptLarge))
      path = FK_PATH_CLUSTER;
    else
      path = FK_PATH_TWOPHASE;
  }
  fk_softmax_plan p = {path, 0, 0, 1};
  switch (path) {
    case FK_PATH_WARP: {
      int vpt = 1;
      while (vpt < 8 && warp_cap(dtype, vpt) < cols) vpt *= 2;
      if (warp_cap(dtype, vpt) < cols) return FK_ERR_INVALID_ARG;
      p.threads = kWarpThreads;
      p.vpt = vpt;
      break;
    }
    case FK_PATH_CTA: {
      int t = 128;
      while (t < 1024 && block_cap(t, ept_cta) < cols) t *= 2;
      if (block_cap(t, ept_cta) < cols) return FK_ERR_INVALID_ARG;
      p.threads = t;
      p.vpt = ept_cta / vec;
      break;
    }
    case FK_PATH_CLUSTER: {
      // 64 values per thread; the smallest block (128, 256, then 512
      // threads) whose cluster of at most 16 holds the row
      int t = 128;
      size_t k = ceil_div(cols, block_cap(t, kClusterEpt));
      while (k > static_cast<size_t>(kMaxCluster) && t < 512) {
        t *= 2;
        k = ceil_div(cols, block_cap(t, kClusterEpt));
      }
      if (k < 2) k = 2;
      if (k > static_cast<size_t>(kMaxCluster)) return FK_ERR_INVALID_ARG;
      p.threads = t;
      p.vpt = kClusterEpt / vec;
      p.cluster = static_cast<int>(k);
      break;
    }
    case FK_PATH_TWOPHASE: {
      // enough blocks that each streams at most ~4 chunks, capped at 16
      const size_t chunk = static_cast<size_t>(kTwoPhaseThreads) * kTwoPhaseElemsPerThread;
      size_t k = ceil_div(cols, chunk * 4);
      if (k < 1) k = 1;
      if (k > static_cast<size_t>(kMaxCluster)) k = kMaxCluster;
      p.threads = kTwoPhaseThreads;
      p.vpt = kTwoPhaseElemsPerThread / vec;
      p.cluster = static_cast<int>(k);
      break;
    }
    default:
      return FK_ERR_INVALID_ARG;
  }
  *out = p;
  return FK_OK;
}

fk_status check_plan(size_t cols, int dtype, const fk_softmax_plan& in, fk_softmax_plan* out) {
  if (!valid_dtype(dtype)) return FK_ERR_UNSUPPORTED_DTYPE;
  const int vec = vec_elems(dtype);
  fk_softmax_plan d;
  const fk_status st = plan_softmax(1, cols, dtype, in.path, &d);
  if (st != FK_OK) {
    // the default for this path may not hold cols, but an explicit plan could
    if (in.path != FK_PATH_CTA && in.path != FK_PATH_CLUSTER) return st;
    d.path = in.path;
    d.threads = in.path == FK_PATH_CLUSTER ? 512 : 1024;
    d.vpt = (in.path == FK_PATH_CLUSTER ? kClusterEpt : kBlockEptLarge) / vec;
    d.cluster = in.path == FK_PATH_CLUSTER ? kMaxCluster : 1;
  }
  fk_softmax_plan p = d;
  if (in.threads != 0) p.threads = in.threads;
  if (in.vpt != 0) p.vpt = in.vpt;
  if (in.cluster != 0) p.cluster = in.cluster;
  switch (p.path) {
    case FK_PATH_WARP:
      if (p.threads != kWarpThreads || p.cluster != 1) return FK_ERR_INVALID_ARG;
      if (p.vpt != 1 && p.vpt != 2 && p.vpt != 4 && p.vpt != 8) return FK_ERR_INVALID_ARG;
      if (warp_cap(dtype, p.vpt) < cols) return FK_ERR_INVALID_ARG;
      break;
    case FK_PATH_CTA:
      if (!block_threads_ok(p.threads) || p.cluster != 1) return FK_ERR_INVALID_ARG;
      if (!ept_ok(p.vpt * vec)) return FK_ERR_INVALID_ARG;
      if (block_cap(p.threads, p.vpt * vec) < cols) return FK_ERR_INVALID_ARG;
      break;
    case FK_PATH_CLUSTER:
      if (!block_threads_ok(p.threads) || p.cluster < 2 || p.cluster > kMaxCluster)
        return FK_ERR_INVALID_ARG;
      if (!cluster_ept_ok(p.vpt * vec, p.threads)) return FK_ERR_INVALID_ARG;
      // each block's slice, ceil(vectors / cluster), must fit its registers
      if (ceil_div(ceil_div(cols, vec), p.cluster) * vec > block_cap(p.threads, p.vpt * vec))
        return FK_ERR_INVALID_ARG;
      break;
    case FK_PATH_TWOPHASE:
      if (p.threads != kTwoPhaseThreads || p.vpt != kTwoPhaseElemsPerThread / vec)
        return FK_ERR_INVALID_ARG;
      if (p.cluster < 1 || p.cluster > kMaxCluster) return FK_ERR_INVALID_ARG;
      break;
    default:
      return FK_ERR_INVALID_ARG;
  }
  *out = p;
  return FK_OK;
}

}  // namespace fk
