/*
 * fk.h -- C ABI of libfk: fused memory-bound operators for NVIDIA B200 (sm_100a).
 *
 * The two core operators are each one kernel that reads every input element
 * once from HBM and writes every output element once (the fusion argument
 * of "Lecture 6: GPU Kernels and Triton", cs336.sjfarmltd.com, section 1.1:
 * one read plus one write instead of a read and a write per separate op):
 *
 *   fk_gelu_tanh     y = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
 *                    -- CS336 lecture-6 notes (kyc001.github.io), section 4.2.
 *   fk_softmax_rows  y[r, j] = exp(x[r, j] - m_r) / sum_k exp(x[r, k] - m_r),
 *                    m_r = max_k x[r, k], over the last axis of a row-major
 *                    [rows, cols] matrix -- lecture 6, section 7.2 (two-pass
 *                    form; the running max/sum merge of the same section is
 *                    used where one row is split across thread blocks), and
 *                    the lecture-6 notes, section 5.2 (row max, exponentials
 *                    and sum, normalise).
 *
 * Around them, the same one-pass design for the neighbouring steps the
 * lecture builds on: fk_gelu (both GELU forms, fp32 or bf16),
 * fk_softmax_rows_causal (scaled, causally masked softmax with the mask made
 * in the kernel), fk_layernorm_rows (LayerNorm, optional affine and GELU
 * epilogue), and fk_attention_fwd (attention forward on the tensor cores,
 * the Flash-Attention computation of lecture 6, sections 7.3 and 8).
 *
 * Conventions common to every entry point
 * ---------------------------------------
 * Memory:    every pointer is caller-owned memory that the current CUDA
 *            device can access (cudaMalloc / torch tensors, managed or
 *            mapped pinned host memory).  Pageable host memory is rejected
 *            (FK_ERR_INVALID_ARG).  libfk holds no handles and keeps no state
 *            besides a per-device properties cache.  The only allocation it
 *            ever makes is the workspace of the split path (FK_PATH_SPLIT:
 *            very long rows, few of them), a few KiB to at most 8 MiB taken
 *            stream-ordered on the caller's stream from a private memory pool
 *            of the library (which keeps up to 64 MiB reserved between calls)
 *            and released on the same stream; fk_softmax_rows_ws takes a
 *            caller-provided workspace instead and allocates nothing.
 * Layout:    contiguous; softmax rows are row-major with row stride = cols.
 * Streams:   `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *            default stream).  Calls are asynchronous: the kernel is enqueued
 *            and the call returns without synchronising.
 * Aliasing:  x == y (in place) is allowed; any other overlap of the input and
 *            output ranges is rejected.
 * Errors:    all argument checks run on the host before anything is
 *            enqueued; a failing check returns its code and launches nothing.
 *            A zero-sized problem returns FK_OK and launches nothing (NULL
 *            pointers are then allowed).  A launch failure returns
 *            FK_ERR_CUDA (the CUDA error code is kept per host thread, see
 *            fk_last_cuda_error).  Errors of the asynchronous execution
 *            surface at the caller's next synchronisation.  Device code never
 *            traps, asserts or prints.
 * Device:    kernels are built for sm_100a only; any other device returns
 *            FK_ERR_UNSUPPORTED_DEVICE.
 * Threads:   every entry point may be called concurrently from several host
 *            threads.
 */
#ifndef FK_H
#define FK_H

#include <stddef.h>

/* Exported entry points keep default visibility even when the library is
 * built with -fvisibility=hidden. */
#if defined(__GNUC__)
#define FK_API __attribute__((visibility("default")))
#else
#define FK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fk_status {
    FK_OK = 0,
    FK_ERR_INVALID_ARG = 1,        /* NULL pointer, bad size/overflow, misalignment, overlap, bad plan */
    FK_ERR_UNSUPPORTED_DTYPE = 2,  /* dtype is not one of fk_dtype */
    FK_ERR_UNSUPPORTED_DEVICE = 3, /* no CUDA device, or not compute capability 10.0 (sm_100a) */
    FK_ERR_CUDA = 4                /* a CUDA runtime call or the launch failed */
} fk_status;

typedef enum fk_dtype {
    FK_F32 = 0,  /* IEEE binary32 */
    FK_BF16 = 1  /* bfloat16 (8-bit exponent, 7-bit fraction); math in fp32, output rounded to nearest even */
} fk_dtype;

/*
 * fk_gelu_tanh -- elementwise GELU, tanh form (lecture-6 notes, section 4.2).
 *   x  [in]  n fp32 values, device-accessible, 4-byte aligned.
 *   y  [out] n fp32 values, same constraints; y == x allowed.
 *   n        element count (0 = no-op).
 *   stream   cudaStream_t as void*.
 * Arithmetic in fp32: y is within 2e-6 of the exact (double) value for every
 * finite x; GELU(+inf) = +inf, GELU(-inf) = -0, GELU(NaN) = NaN.
 * 16-byte aligned x and y (same offset mod 16) take the 128-bit vector path;
 * any other alignment is still correct.
 */
FK_API fk_status fk_gelu_tanh(const float *x, float *y, size_t n, void *stream);

/* GELU forms of fk_gelu. */
typedef enum fk_gelu_kind {
    FK_GELU_TANH = 0, /* 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) (lecture-6 notes, section 4.2) */
    FK_GELU_ERF = 1   /* x Phi(x), the exact form the tanh one approximates */
} fk_gelu_kind;

/*
 * fk_gelu -- elementwise GELU of either form, fp32 or bf16 in and out.
 *   x  [in]  n values of `dtype`, device-accessible, aligned to the element size.
 *   y  [out] n values of the same dtype; y == x allowed.
 *   n        element count (0 = no-op).
 *   dtype    FK_F32 or FK_BF16 (bf16: computed in fp32, rounded to nearest even).
 *   kind     an fk_gelu_kind.
 *   stream   cudaStream_t as void*.
 * Accuracy: fp32 within 2e-6 absolute of the exact value; bf16 within 1 ulp
 * of the correctly rounded value (subnormal outputs included).  GELU(+inf) =
 * +inf, GELU(-inf) = -0, GELU(NaN) = NaN.  fk_gelu_tanh(x, y, n, s) is
 * fk_gelu(x, y, n, FK_F32, FK_GELU_TANH, s).
 */
FK_API fk_status fk_gelu(const void *x, void *y, size_t n, int dtype, int kind, void *stream);

/*
 * fk_copy -- the bandwidth reference: a plain 16-byte streaming copy with
 * the GELU kernel's access pattern (no arithmetic).  The fused kernels are
 * reported against it (the lectures' bandwidth-utilisation metric).
 *   src, dst  device memory, 16-byte aligned, not overlapping.
 *   bytes     a multiple of 16 (0 = no-op).
 * FK_ERR_INVALID_ARG for misalignment, overlap or a size outside either
 * allocation.
 */
FK_API fk_status fk_copy(const void *src, void *dst, size_t bytes, void *stream);

/*
 * fk_softmax_rows -- softmax over each row of a row-major [rows, cols]
 * matrix (lecture 6, section 7.2; lecture-6 notes, section 5.2).
 *   x      [in]  rows*cols elements of `dtype`, device-accessible, aligned to
 *                the element size.
 *   y      [out] rows*cols elements of the same dtype; y == x allowed.
 *   rows, cols   matrix shape (either 0 = no-op).
 *   dtype  an fk_dtype; input and output share it.
 *   stream cudaStream_t as void*.
 * Arithmetic: fp32 for both dtypes (bf16 is widened exactly, accumulated in
 * fp32, rounded to nearest even on store).  Each input element is read from
 * HBM once and each output written once, except for rows longer than a
 * thread-block cluster holds on chip (over 524288 columns of either dtype),
 * which are read twice: by FK_PATH_SPLIT (every chunk of a row in its own
 * block, (max, sum) partials in a workspace, see above) when there are fewer
 * than 4 rows or the rows have 4194304 columns or more, else by
 * FK_PATH_TWOPHASE (one cluster per row).
 * -inf inputs give exactly 0; a row that is all -inf, or holds a NaN or a
 * +inf, gives NaN throughout.
 */
FK_API fk_status fk_softmax_rows(const void *x, void *y, size_t rows, size_t cols, int dtype, void *stream);

/* Kernel paths of fk_softmax_rows. */
typedef enum fk_softmax_path {
    FK_PATH_AUTO = 0,     /* let fk_softmax_rows_plan choose */
    FK_PATH_WARP = 1,     /* one warp per row, row held in registers */
    FK_PATH_CTA = 2,      /* one thread block per row, row held in registers */
    FK_PATH_CLUSTER = 3,  /* one thread-block cluster per row, slices in registers,
                             (max, sum) partials merged over distributed shared memory */
    FK_PATH_TWOPHASE = 4, /* one cluster per row, streamed twice: running (max, sum)
                             pass, then normalise pass -- any row length */
    FK_PATH_SPLIT = 5     /* every chunk of every row in its own block: a stats kernel
                             writes each chunk's (max, sum) to a workspace, a normalise
                             kernel merges a row's partials -- any row length, any
                             number of rows, needs workspace */
} fk_softmax_path;

/* A resolved launch plan.  `threads` = threads per block (on FK_PATH_WARP,
 * 32 x the rows one block takes: 32, 64, 128 or 256, chosen from the row
 * count so that few rows still reach every multiprocessor); `vpt` = 16-byte
 * vectors per thread per step; `cluster` = blocks per row for the cluster
 * paths (1 otherwise); `chunks` = blocks per row on the split path (derived
 * from the shape; 1 otherwise). */
typedef struct fk_softmax_plan {
    int path;
    int threads;
    int vpt;
    int cluster;
    int chunks;
} fk_softmax_plan;

/*
 * fk_softmax_rows_plan -- the plan fk_softmax_rows would use (host only,
 * launches nothing, needs no device).
 *   rows, cols, dtype  as for fk_softmax_rows (cols > 0).
 *   path     FK_PATH_AUTO, or a path to force; its threads/vpt/cluster are
 *            then chosen for that path.
 *   out      [out] the plan.
 * Returns FK_ERR_INVALID_ARG when the forced path cannot hold `cols`
 * (WARP/CTA/CLUSTER have fixed on-chip capacities).
 */
FK_API fk_status fk_softmax_rows_plan(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan *out);

/*
 * fk_softmax_rows_ex -- fk_softmax_rows with an explicit plan (tests and
 * tuning).  plan == NULL or plan->path == FK_PATH_AUTO behaves like
 * fk_softmax_rows.  Otherwise every field is validated against the compiled
 * kernel set (threads in {32,64,128,256} for the warp path and
 * {128,256,512,1024} for block paths; cluster in
 * 1..16; vpt fixed per dtype and path) and FK_ERR_INVALID_ARG is returned
 * for a plan that is not built or cannot hold `cols`.  Zero fields take the
 * path's defaults.
 */
FK_API fk_status fk_softmax_rows_ex(const void *x, void *y, size_t rows, size_t cols, int dtype,
                             const fk_softmax_plan *plan, void *stream);

/*
 * fk_softmax_rows_workspace -- device workspace, in bytes, that a softmax
 * call of this shape and plan needs (0 for every path but FK_PATH_SPLIT;
 * at most 8 MiB).  Host only.
 *   plan   NULL or FK_PATH_AUTO = the automatic plan.
 *   bytes  [out]
 */
FK_API fk_status fk_softmax_rows_workspace(size_t rows, size_t cols, int dtype, const fk_softmax_plan *plan,
                                           size_t *bytes);

/*
 * fk_softmax_rows_ws -- fk_softmax_rows_ex with caller-provided workspace;
 * allocates nothing.
 *   workspace        device memory of at least fk_softmax_rows_workspace
 *                    bytes, 8-byte aligned, not overlapping x or y (may be
 *                    NULL when that size is 0).  Its contents on entry do not
 *                    matter; it must not be used by other work until the
 *                    call's kernels have finished on `stream`.
 *   workspace_bytes  its size; too small -> FK_ERR_INVALID_ARG.
 */
FK_API fk_status fk_softmax_rows_ws(const void *x, void *y, size_t rows, size_t cols, int dtype,
                                    const fk_softmax_plan *plan, void *workspace, size_t workspace_bytes,
                                    void *stream);

/*
 * fk_softmax_rows_noalloc -- fk_softmax_rows that never allocates device
 * memory (the lecture pages have no counterpart; this is a library
 * convenience).  For callers that cannot call cudaMalloc or let a library do
 * so: code under a framework that has reserved nearly all device memory for
 * its own allocator, latency-critical loops that cannot afford an allocation
 * call (cudaMalloc may synchronise the device), environments whose policy
 * forbids a library from allocating.
 *   Arguments, plan and results as fk_softmax_rows.  Only the split path
 *   (few or very long rows) needs scratch; here it is a fixed 1 MiB device
 *   array inside the library (131072 (max, sum) pairs), which every GPU that
 *   loads the library holds until the process exits.  Rows are processed in
 *   batches whose partials fit it; a row of more than 2^35 elements (which
 *   would need more than 131072 chunks; a chunk holds at most 262144
 *   elements) returns FK_ERR_INVALID_ARG.  Every check,
 *   including that x and y lie wholly inside device allocations, runs before
 *   the first batch is enqueued, so a call that returns an error has written
 *   nothing.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and keeps it; a lookup
 *   that fails is retried by the next call.  Make that first call before any
 *   stream capture.
 *   All calls on a device share the array and it keeps the last call's
 *   contents (nothing in it needs clearing: each call writes every partial
 *   it reads before reading it).  Calls whose kernels overlap on the GPU --
 *   on different streams without ordering between them -- race on it and
 *   give wrong results; order them (one stream, or events).
 */
FK_API fk_status fk_softmax_rows_noalloc(const void *x, void *y, size_t rows, size_t cols, int dtype,
                                         void *stream);

/*
 * fk_softmax_rows_noalloc_cap -- fk_softmax_rows_noalloc using only the
 * first capacity_pairs (max, sum) pairs of the library's array (1 ..
 * 131072), so that the batching can be exercised on inputs of a few GB: rows
 * run in batches of floor(capacity_pairs / chunks) rows.  A capacity that
 * cannot hold one row's chunks, or the chunks of the full batch or of the
 * shorter last batch as each is planned, returns FK_ERR_INVALID_ARG before
 * anything is enqueued; capacity_pairs outside 1 .. 131072 likewise.
 * Otherwise as fk_softmax_rows_noalloc (same array, same ordering rules).
 */
FK_API fk_status fk_softmax_rows_noalloc_cap(const void *x, void *y, size_t rows, size_t cols, int dtype,
                                             size_t capacity_pairs, void *stream);

/*
 * fk_softmax_rows_causal -- scaled, causally masked row softmax: the score
 * step of causal attention (lecture 6, "GPU Kernels and Triton", section 8:
 * scores times 1/sqrt(d_k), -inf where the key position is after the query
 * position, then softmax) in one pass, with the mask generated in the kernel
 * instead of read from an -inf tensor.  Row r keeps the columns
 *     j <= q(r) = (r mod period) + offset
 * (every column when period == 0) and gets
 *     y[r, j] = exp(scale (x[r, j] - m)) / sum_{i <= q(r)} exp(scale (x[r, i] - m)),
 *     m = max_{i <= q(r)} x[r, i],
 * and y[r, j] = 0 for j > q(r).  Masked inputs are never read (they may hold
 * anything), so a causal [T, T] score block moves about 25% fewer bytes than
 * softmax over an explicitly masked tensor.
 *   x, y, rows, cols, dtype, stream   as for fk_softmax_rows.
 *   scale   finite and > 0 (e.g. 1/sqrt(d_k)); applied in fp32 as
 *           scale * log2(e) rounded once.
 *   period  the rows per query block: for scores laid out [batch, heads, T_q,
 *           T_k] as rows of T_k columns, period = T_q; 0 = no mask (a scaled
 *           softmax).
 *   offset  the query position of each block's first row: 0 when queries and
 *           keys start together, T_k - T_q for the last T_q positions of a
 *           T_k-long sequence.
 * Paths, special values and errors as fk_softmax_rows (a kept -inf gives 0;
 * every row keeps at least column 0, so no row is empty).  Values with
 * |scale * x| beyond about 2^126 overflow the fp32 exponent arithmetic (NaN
 * in that row).  scale not finite or <= 0 -> FK_ERR_INVALID_ARG.
 */
FK_API fk_status fk_softmax_rows_causal(const void *x, void *y, size_t rows, size_t cols, int dtype, float scale,
                                        size_t period, size_t offset, void *stream);

/* Flags of fk_softmax_rows_causal_ex. */
#define FK_SOFTMAX_SKIP_MASKED 1u /* do not store masked outputs: each masked output is then
                                     either left as it was or set to 0 (0 where it shares a
                                     16-byte vector with a kept output).  For consumers that
                                     never read the masked region: the output's write traffic
                                     halves along with the reads. */

/* fk_softmax_rows_causal with flags (0 or FK_SOFTMAX_SKIP_MASKED; other
 * bits -> FK_ERR_INVALID_ARG) and an explicit plan, as fk_softmax_rows_ex. */
FK_API fk_status fk_softmax_rows_causal_ex(const void *x, void *y, size_t rows, size_t cols, int dtype,
                                           float scale, size_t period, size_t offset, unsigned int flags,
                                           const fk_softmax_plan *plan, void *stream);

/* Epilogues of fk_layernorm_rows. */
typedef enum fk_epilogue {
    FK_EPILOGUE_NONE = 0,
    FK_EPILOGUE_GELU_TANH = 1, /* GELU, tanh form, of the normalised value */
    FK_EPILOGUE_GELU_ERF = 2   /* GELU, exact form */
} fk_epilogue;

/*
 * fk_layernorm_rows -- LayerNorm over each row of a row-major [rows, cols]
 * matrix, optionally followed by GELU, in one pass over HBM: the
 * normalisation and activation of the fused LayerNorm -> Linear -> GELU
 * example (lecture 6, "GPU Kernels and Triton", sections 6.1-6.2, where it
 * is F.layer_norm over the last axis).
 *     mean = sum_j x_j / cols,   var = sum_j (x_j - mean)^2 / cols (biased),
 *     y_j  = epilogue( (x_j - mean) / sqrt(var + eps) * gamma_j + beta_j ).
 *   x, y    rows*cols elements of `dtype` (FK_F32 or FK_BF16), device
 *           memory; y == x allowed, other overlap rejected.
 *   gamma, beta  fp32 device arrays of cols values, or NULL (1 and 0); must
 *           not overlap y.  16-byte alignment (with 16-byte-multiple rows)
 *           selects the vector path; any 4-byte alignment works.
 *   eps     finite, >= 0 (PyTorch's default is 1e-5).
 *   epilogue  an fk_epilogue.
 * Arithmetic in fp32 (bf16 widened exactly, rounded to nearest even on
 * store).  The row is read once and written once up to 32768 columns; longer
 * rows are read twice.  A row holding a NaN or an infinity gives NaN
 * throughout; a constant row gives beta (or NaN when eps == 0).
 * Errors: FK_ERR_INVALID_ARG for bad pointers, overlap, eps < 0 or not
 * finite, or an unknown epilogue.
 */
FK_API fk_status fk_layernorm_rows(const void *x, void *y, const float *gamma, const float *beta, size_t rows,
                                   size_t cols, int dtype, float eps, int epilogue, void *stream);

/* The plan fk_layernorm_rows would use (host only; path FK_PATH_AUTO or one
 * to force: FK_PATH_WARP, FK_PATH_CTA or FK_PATH_TWOPHASE). */
FK_API fk_status fk_layernorm_rows_plan(size_t rows, size_t cols, int dtype, int path, fk_softmax_plan *out);

/* fk_layernorm_rows with an explicit plan: FK_PATH_WARP, FK_PATH_CTA (as for
 * softmax) or FK_PATH_TWOPHASE (one 512-thread block per row, streamed
 * twice); NULL or FK_PATH_AUTO = the automatic choice. */
FK_API fk_status fk_layernorm_rows_ex(const void *x, void *y, const float *gamma, const float *beta,
                                      size_t rows, size_t cols, int dtype, float eps, int epilogue,
                                      const fk_softmax_plan *plan, void *stream);

/*
 * fk_attention_fwd -- attention forward on the tensor cores, the computation
 * Flash Attention tiles (lecture 6, "GPU Kernels and Triton", sections 7.3
 * and 8):
 *     O = softmax(scale * Q K^T  [+ causal mask: key j > query i is -inf]) V
 * for bh independent (batch, head) slices; S and P stay on chip (tensor
 * memory), with the running max / sum of section 7.2.
 *   q, k, v  [bh, t, d] bf16, contiguous, device memory, 16-byte aligned.
 *   o        [bh, t, d] bf16 output; must not overlap q, k or v.
 *   t        a multiple of 128, at most 128 * 65535 (queries and keys per
 *            slice); d = 64 or 128.
 *   causal   0 or 1.
 *   scale    finite, > 0 (e.g. 1 / sqrt(d)).
 * Arithmetic: S and the O accumulator in fp32 (tcgen05, TMEM), P rounded to
 * bf16 for the second product, O rounded to bf16 at the end.
 * Errors: FK_ERR_INVALID_ARG for a shape or argument outside the above,
 * bh * t >= 2^31, bad pointers or overlap; FK_ERR_CUDA if the kernel cannot
 * be launched (including a build whose register allocation cannot fund the
 * kernel's warp-specialised register split, which it checks before
 * launching).  A wait that gives up (see fk_wait_timeouts) leaves that
 * block of O unwritten.
 */
FK_API fk_status fk_attention_fwd(const void *q, const void *k, const void *v, void *o, size_t bh, size_t t,
                                  size_t d, int causal, float scale, void *stream);

/*
 * fk_wait_timeouts -- health check of the cluster paths.  Blocks of a
 * cluster exchange their partial (max, sum) through mbarriers; every such
 * wait is bounded in time (1 s) and a wait that gives up is counted instead
 * of hanging the GPU (the row is then not valid).
 *   count  [out] number of threads whose wait gave up on the current device
 *          since the library was loaded or last reset.
 *   reset  nonzero: set the count back to 0 after reading it.
 * Synchronous; call after the work of interest has completed.  A nonzero
 * count in normal operation means a partner block never arrived.  A call
 * whose wait gave up still returns FK_OK (the give-up happens on the GPU,
 * after the call has returned), so callers that must detect it read this
 * count after synchronising.
 */
FK_API fk_status fk_wait_timeouts(unsigned int *count, int reset);

/*
 * fk_wait_selftest -- launch one block of 32 threads that waits on an
 * mbarrier nothing arrives on, with a limit of timeout_us microseconds
 * (1..10000000); each thread gives up and adds 1 to fk_wait_timeouts.  Tests
 * the give-up path without faulting or hanging the GPU.  Asynchronous on
 * `stream`.
 */
FK_API fk_status fk_wait_selftest(unsigned int timeout_us, void *stream);

/* Static description of a status code (never NULL). */
FK_API const char *fk_status_string(int status);

/* The cudaError_t of the last FK_ERR_CUDA returned on this host thread
 * (0 if none). */
FK_API int fk_last_cuda_error(void);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
FK_API int fk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FK_H */
