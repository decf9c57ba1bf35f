// fk_plan.cpp -- host-only choice of the softmax kernel for a row length.
//
// The capacities follow from the kernels' register budgets:
//   warp     : 32 lanes x VPT 16-byte vectors, VPT in {1, 2, 4, 8}
//              -> up to 1024 fp32 / 2048 bf16 columns; 1 to 8 rows (warps)
//              per block, 2 to 8 by default (see warp_threads_for)
//   block    : 16 or 32 elements per thread (EPT), threads in
//              {128, 256, 512, 1024} -> up to 32768 columns (the automatic
//              plan takes it up to 8192 columns, 256 threads)
//   cluster  : 2..16 blocks of 128..512 threads holding 64 values each
//              -> up to 524288 columns
//   twophase : any length; one cluster per row streams it twice
//   split    : any length; every chunk of every row gets its own block, and a
//              small workspace carries the chunks' (max, sum) partials --
//              the choice for long rows when there are too few rows to give
//              one cluster each and still fill the GPU
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

constexpr int kPlanSmCount = 148;  // B200 multiprocessors: the plans are chosen on the host, without a device

bool warp_threads_ok(int t) { return t == 32 || t == 64 || t == 128 || t == kWarpThreads; }

// Warp path: kWarpRowsPerBlock rows per block, halved (down to two) while the
// grid would leave multiprocessors without a block, so that a few hundred
// rows are spread over the whole GPU rather than a quarter of it.  Measured
// on B200, fp32 rows of 1000 with L2 cleaned: 256 rows take 8.14 us with 8
// rows per block, 6.64 with 2 and 6.87 with 1 (a 1 MB copy: 6.17); 512 rows
// 8.15 with 8, 7.60 with 4; from 768 rows every choice ties.
int warp_threads_for(size_t rows) {
  int r = kWarpRowsPerBlock;
  while (r > 2 && ceil_div(rows, static_cast<size_t>(r)) < static_cast<size_t>(kPlanSmCount)) r /= 2;
  return 32 * r;
}

constexpr size_t kSplitFillBlocks = 148 * 8;     // blocks that fill a B200 several times over
constexpr size_t kSplitMaxIters = 32;             // streamed steps per block at most
constexpr size_t kSplitMaxPartials = size_t{1} << 20;  // workspace: 8 MiB of partials at most
// Long rows (past cluster capacity) use the split path when there are fewer
// than kSplitBelowRows rows, or when rows have kSplitFromCols columns or more;
// otherwise one cluster per row streams it twice.  Measured on B200 (fp32,
// L2 cleaned): at 1M columns the cluster path wins from 4 to 32 rows (e.g.
// 2.18 vs 1.99 TB/s at 8 rows) and they tie from 64 rows; at 4M and 16M
// columns the split path wins at every row count (1.43 vs 0.47 TB/s at one
// row of 4M, 3.05 vs 0.52 at one row of 16M, 4.37 vs 4.18 at 128 rows of 4M).
constexpr size_t kSplitBelowRows = 4;
constexpr size_t kSplitFromCols = size_t{1} << 22;

bool cluster_ept_ok(int ept, int threads) {
  return ept_ok(ept) || (ept == kClusterEpt && threads <= 512);
}

}  // namespace

SplitGeometry split_geometry(size_t rows, size_t cols, int dtype) {
  const size_t vec = static_cast<size_t>(vec_elems(dtype));
  const size_t unit = static_cast<size_t>(kTwoPhaseThreads) * (kTwoPhaseElemsPerThread / vec);  // vectors/step
  const size_t nvec = ceil_div(cols, vec);
  size_t want = ceil_div(kSplitFillBlocks, rows > 0 ? rows : 1);
  const size_t by_len = ceil_div(nvec, unit * kSplitMaxIters);
  if (want < by_len) want = by_len;
  if (want < 1) want = 1;
  SplitGeometry g;
  g.chunk_vecs = ceil_div(ceil_div(nvec, want), unit) * unit;
  g.nchunks = static_cast<unsigned>(ceil_div(nvec, g.chunk_vecs));
  size_t rpl = kSplitMaxPartials / g.nchunks;
  if (rpl < 1) rpl = 1;
  if (rpl > rows) rpl = rows > 0 ? rows : 1;
  g.rows_per_launch = rpl;
  g.ws_bytes = rpl * g.nchunks * 8;
  return g;
}

size_t workspace_bytes(size_t rows, size_t cols, int dtype, const fk_softmax_plan& plan) {
  return plan.path == FK_PATH_SPLIT ? split_geometry(rows, cols, dtype).ws_bytes : 0;
}

fk_status plan_softmax(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out) {
  if (!valid_dtype(dtype)) return FK_ERR_UNSUPPORTED_DTYPE;
  if (out == nullptr || cols == 0) return FK_ERR_INVALID_ARG;
  const int vec = vec_elems(dtype);
  // elements per thread on the block paths: bf16 rows of up to 2048 columns
  // take the small budget (fewer registers, more resident blocks), every
  // other row the large one
  const int ept_cta = (dtype == FK_BF16 && cols <= block_cap(128, kBlockEptSmall)) ? kBlockEptSmall
                                                                                  : kBlockEptLarge;
  if (path == FK_PATH_AUTO) {
    // One block per row up to 256 threads' worth; wider rows go to clusters
    // of small blocks, whose reductions are shorter and whose blocks fit
    // more per SM.  Measured on B200 (256 MiB of rows, L2 cleaned, against a
    // copy): fp32 16384 columns 0.67 with one 512-thread block, 0.99 with
    // clusters of two 128-thread blocks; 32768 columns 0.72 / 0.99 (four);
    // bf16 8192 columns 0.75 with 512 threads x 16 values, 0.98 with 256 x
    // 32; 16384 columns 0.42 / 0.84 (clusters of two); 32768 0.55 / 0.81.
    if (cols <= 1024)
      path = FK_PATH_WARP;
    else if (cols <= block_cap(256, kBlockEptLarge))
      path = FK_PATH_CTA;
    else if (cols <= static_cast<size_t>(kMaxCluster) * block_cap(1024, kBlockEptLarge))
      path = FK_PATH_CLUSTER;
    else if (rows < kSplitBelowRows || cols >= kSplitFromCols)
      path = FK_PATH_SPLIT;
    else
      path = FK_PATH_TWOPHASE;
  }
  fk_softmax_plan p = {path, 0, 0, 1, 1};
  switch (path) {
    case FK_PATH_WARP: {
      int vpt = 1;
      while (vpt < 8 && warp_cap(dtype, vpt) < cols) vpt *= 2;
      if (warp_cap(dtype, vpt) < cols) return FK_ERR_INVALID_ARG;
      p.threads = warp_threads_for(rows);
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
    case FK_PATH_SPLIT: {
      p.threads = kTwoPhaseThreads;
      p.vpt = kTwoPhaseElemsPerThread / vec;
      p.cluster = 1;
      p.chunks = static_cast<int>(split_geometry(rows, cols, dtype).nchunks);
      break;
    }
    default:
      return FK_ERR_INVALID_ARG;
  }
  *out = p;
  return FK_OK;
}

fk_status check_plan(size_t rows, size_t cols, int dtype, const fk_softmax_plan& in, fk_softmax_plan* out) {
  if (!valid_dtype(dtype)) return FK_ERR_UNSUPPORTED_DTYPE;
  const int vec = vec_elems(dtype);
  fk_softmax_plan d;
  const fk_status st = plan_softmax(rows, cols, dtype, in.path, &d);
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
      if (!warp_threads_ok(p.threads) || p.cluster != 1) return FK_ERR_INVALID_ARG;
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
    case FK_PATH_SPLIT:
      // the chunking is derived from the shape; only the defaults are accepted
      if (p.threads != kTwoPhaseThreads || p.vpt != kTwoPhaseElemsPerThread / vec || p.cluster != 1)
        return FK_ERR_INVALID_ARG;
      if (in.chunks != 0 && in.chunks != d.chunks) return FK_ERR_INVALID_ARG;
      p.chunks = d.chunks;
      break;
    default:
      return FK_ERR_INVALID_ARG;
  }
  if (p.path != FK_PATH_SPLIT) p.chunks = 1;
  *out = p;
  return FK_OK;
}

fk_status plan_layernorm(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan* out) {
  if (!valid_dtype(dtype)) return FK_ERR_UNSUPPORTED_DTYPE;
  if (out == nullptr || cols == 0) return FK_ERR_INVALID_ARG;
  if (path == FK_PATH_AUTO) {
    if (cols <= 1024)
      path = FK_PATH_WARP;
    else if (cols <= block_cap(1024, kBlockEptLarge))
      path = FK_PATH_CTA;
    else
      path = FK_PATH_TWOPHASE;
  }
  if (path == FK_PATH_WARP) return plan_softmax(rows, cols, dtype, path, out);
  if (path == FK_PATH_CTA) {
    // 32 values per thread (the row stays packed in registers), except for
    // rows that 128 threads hold with 16.  Measured on B200, 65536 rows of
    // 4096 with gamma / beta: fp32 6595 GB/s at 128 x 32 against 6473 at
    // 256 x 16 (6242 against 5608 with the GELU epilogue); bf16 4855 against
    // 3692.
    const int ept = cols <= block_cap(128, kBlockEptSmall) ? kBlockEptSmall : kBlockEptLarge;
    int t = 128;
    while (t < 1024 && block_cap(t, ept) < cols) t *= 2;
    if (block_cap(t, ept) < cols) return FK_ERR_INVALID_ARG;
    *out = fk_softmax_plan{FK_PATH_CTA, t, ept / vec_elems(dtype), 1, 1};
    return FK_OK;
  }
  if (path != FK_PATH_TWOPHASE) return FK_ERR_INVALID_ARG;
  *out = fk_softmax_plan{FK_PATH_TWOPHASE, kTwoPhaseThreads, kTwoPhaseElemsPerThread / vec_elems(dtype), 1, 1};
  return FK_OK;
}

fk_status check_layernorm_plan(size_t rows, size_t cols, int dtype, const fk_softmax_plan& in,
                               fk_softmax_plan* out) {
  if (!valid_dtype(dtype)) return FK_ERR_UNSUPPORTED_DTYPE;
  if (in.path == FK_PATH_WARP || in.path == FK_PATH_CTA) return check_plan(rows, cols, dtype, in, out);
  if (in.path != FK_PATH_TWOPHASE) return FK_ERR_INVALID_ARG;
  fk_softmax_plan p;
  const fk_status st = plan_layernorm(rows, cols, dtype, FK_PATH_TWOPHASE, &p);
  if (st != FK_OK) return st;
  // the streaming kernel has one shape: 512 threads, one block per row
  if ((in.threads != 0 && in.threads != p.threads) || (in.vpt != 0 && in.vpt != p.vpt) ||
      (in.cluster != 0 && in.cluster != 1))
    return FK_ERR_INVALID_ARG;
  *out = p;
  return FK_OK;
}

void set_period_division(SoftmaxScaling* sc, size_t rows) {
  sc->magic = 0;
  sc->shift1 = 0;
  sc->shift2 = 0;
  sc->fast32 = 0;
  const uint64_t d = sc->period;
  if (d == 0 || d > 0xffffffffull || rows > 0xffffffffull) return;
  // l = ceil(log2 d); magic = floor(2^32 (2^l - d) / d) + 1, which is < 2^32
  unsigned l = 0;
  while ((uint64_t{1} << l) < d) ++l;
  sc->magic = static_cast<uint32_t>((((uint64_t{1} << l) - d) << 32) / d + 1);
  sc->shift1 = l < 1 ? l : 1;
  sc->shift2 = l > 1 ? l - 1 : 0;
  sc->fast32 = 1;
}

}  // namespace fk
