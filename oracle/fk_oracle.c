/*
 * fk_oracle.c -- plain CPU oracle for the two fused memory-bound operators.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * reference that the CUDA library is checked against.  It shares no code,
 * header, constant or helper with the CUDA library (memory_bound_fk_b200/),
 * and the CUDA library never calls it.  Only tests/, the smoke check in
 * __graft_entry__.py and the cpu_baseline / reference legs of bench.py may
 * load it.
 *
 * Everything is computed in IEEE double precision, straight from the
 * definitions, with no blocking, fusion or reordering:
 *
 *   GELU, tanh form -- "GPU Kernels" lecture-6 notes (kyc001.github.io,
 *   CS336 lecture 6), section 4.2 "GELU":
 *       GELU(x) = 0.5 x (1 + tanh( sqrt(2/pi) (x + 0.044715 x^3) ))
 *   The constant 0.044715 is the decimal printed there; sqrt(2/pi) is
 *   evaluated in double at run time.
 *
 *   Row softmax -- "Lecture 6: GPU Kernels and Triton" (cs336.sjfarmltd.com),
 *   section 7.2 "Online Softmax", the two-pass form: first the row maximum
 *   and the sum of exp(x - max), then exp(x - max) / sum; and the
 *   lecture-6 notes (kyc001.github.io), section 5.2: one row at a time,
 *   max, then exponentials and their sum, then normalise.
 *
 * Readings taken where the pages are silent (each also listed in the
 * design notes):
 *   - the softmax axis is the last one of a row-major [rows, cols] matrix;
 *   - GELU(+inf) = +inf and GELU(-inf) = -0 (the limits); the literal
 *     formula would give (-inf) * 0 = NaN at -inf;
 *   - a row that is entirely -inf gives NaN everywhere (0/0); a row that
 *     holds a NaN or a +inf gives NaN everywhere (inf - inf);
 *   - the row sum uses Neumaier's compensated summation so that the double
 *     result is accurate to a few units in the last place for any length;
 *   - results are rounded once, double -> target type, round to nearest
 *     even (the bf16 rounding works from the double bits directly, so there
 *     is no intermediate fp32 rounding).
 *
 *   LayerNorm (+ GELU) and the scaled, causally masked softmax: see their
 *   sections below.
 *
 * Rows (and GELU element ranges) are split across POSIX threads; each row
 * is computed by exactly one thread with the same sequential arithmetic,
 * so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Scalar definitions                                                  */
/* ------------------------------------------------------------------ */

/* GELU, tanh approximation, lecture-6 notes section 4.2:
 * 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3).
 * For x < 0 the sum 1 + tanh(u) cancels -- in double it is 0 once u < -19,
 * while GELU(-8) is about -3e-21 -- so there it is taken through the exact
 * identity 1 + tanh(u) = 2 e^(2u) / (1 + e^(2u)), which keeps the result
 * accurate relative to itself down to double's underflow. */
double oracle_gelu_tanh(double x)
{
    if (isinf(x))
        return x > 0.0 ? x : -0.0; /* limits at +-inf */
    const double k = sqrt(2.0 / M_PI);
    const double u = k * (x + 0.044715 * x * x * x);
    if (x >= 0.0)
        return 0.5 * x * (1.0 + tanh(u));
    const double e = exp(2.0 * u); /* in [0, 1) for x < 0; NaN stays NaN */
    return 0.5 * x * (2.0 * e / (1.0 + e));
}

/* GELU, exact form: x * Phi(x), Phi the standard normal distribution
 * function, Phi(x) = erfc(-x / sqrt(2)) / 2 -- the definition the tanh form
 * approximates (the lecture's PyTorch fusion example calls gelu with its
 * default, exact form).  erfc keeps Phi accurate in the far negative tail. */
double oracle_gelu_erf(double x)
{
    if (isinf(x))
        return x > 0.0 ? x : -0.0; /* limits at +-inf */
    return x * 0.5 * erfc(-x / sqrt(2.0));
}

/* Softmax of one row, in place of nothing: reads x[0..n), writes y[0..n).
 * Two passes, as the lecture's section 7.2 states the standard algorithm. */
static void softmax_row_f64(const double *x, double *y, size_t n)
{
    if (n == 0)
        return;
    /* pass 1a: row maximum (a NaN never compares greater, so it is skipped
     * here and then poisons the sum below) */
    double m = -INFINITY;
    for (size_t j = 0; j < n; ++j)
        if (x[j] > m)
            m = x[j];
    /* pass 1b: s = sum_j exp(x_j - m), Neumaier-compensated */
    double s = 0.0, c = 0.0;
    for (size_t j = 0; j < n; ++j) {
        const double e = exp(x[j] - m);
        y[j] = e;
        const double t = s + e;
        if (fabs(s) >= fabs(e))
            c += (s - t) + e;
        else
            c += (e - t) + s;
        s = t;
    }
    s = s + c;
    /* pass 2: normalise */
    for (size_t j = 0; j < n; ++j)
        y[j] = y[j] / s;
}

/* ------------------------------------------------------------------ */
/* Rounding helpers (double -> fp32 / bf16, round to nearest even)      */
/* ------------------------------------------------------------------ */

float oracle_round_to_f32(double v)
{
    /* C's double -> float conversion rounds to nearest even under the
     * default floating-point environment. */
    return (float)v;
}

/* bf16: 1 sign bit, 8 exponent bits (same range as fp32), 7 fraction bits.
 * Normal numbers carry 8 significant bits; the subnormal quantum is 2^-133.
 * Round the double directly to that grid, ties to even. */
uint16_t oracle_round_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    const int neg = signbit(v) ? 1 : 0;
    const double a = fabs(v);
    uint16_t bits;
    if (isinf(a)) {
        bits = 0x7F80;
    } else if (a == 0.0) {
        bits = 0;
    } else {
        int e;
        (void)frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) -> a in [2^(e-1), 2^e) */
        int q_exp = (e - 1) - 7; /* quantum of an 8-significant-bit number */
        if (q_exp < -133)
            q_exp = -133; /* subnormal range */
        const double scaled = ldexp(a, -q_exp); /* exact: power-of-two scale */
        double r = floor(scaled);
        const double frac = scaled - r; /* exact */
        if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
            r += 1.0;
        const double rounded = ldexp(r, q_exp); /* exact */
        if (rounded >= 0x1p128) {
            bits = 0x7F80; /* overflow to infinity */
        } else {
            /* rounded is representable in bf16, hence in fp32 exactly */
            const float f = (float)rounded;
            uint32_t u;
            memcpy(&u, &f, sizeof u);
            bits = (uint16_t)(u >> 16);
        }
    }
    return (uint16_t)(bits | (neg ? 0x8000 : 0));
}

double oracle_bf16_to_f64(uint16_t b)
{
    const uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* Threading: split [0, count) into nthreads contiguous ranges          */
/* ------------------------------------------------------------------ */

typedef void (*range_fn)(void *ctx, size_t begin, size_t end);

typedef struct {
    range_fn fn;
    void *ctx;
    size_t begin, end;
} range_job;

static void *range_job_run(void *p)
{
    range_job *j = (range_job *)p;
    j->fn(j->ctx, j->begin, j->end);
    return NULL;
}

static void parallel_ranges(range_fn fn, void *ctx, size_t count, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if ((size_t)nthreads > count)
        nthreads = count > 0 ? (int)count : 1;
    if (nthreads == 1) {
        fn(ctx, 0, count);
        return;
    }
    pthread_t *tid = (pthread_t *)calloc((size_t)nthreads, sizeof *tid);
    range_job *jobs = (range_job *)calloc((size_t)nthreads, sizeof *jobs);
    int *started = (int *)calloc((size_t)nthreads, sizeof *started);
    const size_t per = count / (size_t)nthreads, extra = count % (size_t)nthreads;
    size_t at = 0;
    for (int t = 0; t < nthreads; ++t) {
        const size_t len = per + ((size_t)t < extra ? 1 : 0);
        jobs[t].fn = fn;
        jobs[t].ctx = ctx;
        jobs[t].begin = at;
        jobs[t].end = at + len;
        at += len;
        started[t] = (pthread_create(&tid[t], NULL, range_job_run, &jobs[t]) == 0);
        if (!started[t]) /* could not start a thread: do its share here */
            fn(ctx, jobs[t].begin, jobs[t].end);
    }
    for (int t = 0; t < nthreads; ++t)
        if (started[t])
            pthread_join(tid[t], NULL);
    free(started);
    free(jobs);
    free(tid);
}

/* ------------------------------------------------------------------ */
/* GELU over arrays                                                     */
/* ------------------------------------------------------------------ */

typedef struct {
    const void *x;
    void *y;
} gelu_ctx;

static void gelu_f64_range(void *p, size_t b, size_t e)
{
    gelu_ctx *c = (gelu_ctx *)p;
    const double *x = (const double *)c->x;
    double *y = (double *)c->y;
    for (size_t i = b; i < e; ++i)
        y[i] = oracle_gelu_tanh(x[i]);
}

static void gelu_f32_range(void *p, size_t b, size_t e)
{
    gelu_ctx *c = (gelu_ctx *)p;
    const float *x = (const float *)c->x;
    float *y = (float *)c->y;
    for (size_t i = b; i < e; ++i)
        y[i] = oracle_round_to_f32(oracle_gelu_tanh((double)x[i]));
}

static void gelu_erf_f64_range(void *p, size_t b, size_t e)
{
    gelu_ctx *c = (gelu_ctx *)p;
    const double *x = (const double *)c->x;
    double *y = (double *)c->y;
    for (size_t i = b; i < e; ++i)
        y[i] = oracle_gelu_erf(x[i]);
}

/* exact (erf) GELU, double in, double out */
void oracle_gelu_erf_f64(const double *x, double *y, size_t n, int nthreads)
{
    gelu_ctx c = {x, y};
    parallel_ranges(gelu_erf_f64_range, &c, n, nthreads);
}

/* double in, double out (no rounding) */
void oracle_gelu_tanh_f64(const double *x, double *y, size_t n, int nthreads)
{
    gelu_ctx c = {x, y};
    parallel_ranges(gelu_f64_range, &c, n, nthreads);
}

/* fp32 in, computed in double, rounded once to fp32 */
void oracle_gelu_tanh_f32(const float *x, float *y, size_t n, int nthreads)
{
    gelu_ctx c = {x, y};
    parallel_ranges(gelu_f32_range, &c, n, nthreads);
}

/* ------------------------------------------------------------------ */
/* Row softmax over matrices                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    const void *x;
    void *y;
    size_t cols;
} softmax_ctx;

static void softmax_f64_range(void *p, size_t b, size_t e)
{
    softmax_ctx *c = (softmax_ctx *)p;
    const double *x = (const double *)c->x;
    double *y = (double *)c->y;
    for (size_t r = b; r < e; ++r)
        softmax_row_f64(x + r * c->cols, y + r * c->cols, c->cols);
}

static void softmax_f32_range(void *p, size_t b, size_t e)
{
    softmax_ctx *c = (softmax_ctx *)p;
    const float *x = (const float *)c->x;
    float *y = (float *)c->y;
    double *xin = (double *)malloc(c->cols * sizeof(double) + 1);
    double *yout = (double *)malloc(c->cols * sizeof(double) + 1);
    for (size_t r = b; r < e; ++r) {
        const float *xr = x + r * c->cols;
        float *yr = y + r * c->cols;
        for (size_t j = 0; j < c->cols; ++j)
            xin[j] = (double)xr[j];
        softmax_row_f64(xin, yout, c->cols);
        for (size_t j = 0; j < c->cols; ++j)
            yr[j] = oracle_round_to_f32(yout[j]);
    }
    free(yout);
    free(xin);
}

static void softmax_bf16_range(void *p, size_t b, size_t e)
{
    softmax_ctx *c = (softmax_ctx *)p;
    const uint16_t *x = (const uint16_t *)c->x;
    uint16_t *y = (uint16_t *)c->y;
    double *xin = (double *)malloc(c->cols * sizeof(double) + 1);
    double *yout = (double *)malloc(c->cols * sizeof(double) + 1);
    for (size_t r = b; r < e; ++r) {
        const uint16_t *xr = x + r * c->cols;
        uint16_t *yr = y + r * c->cols;
        for (size_t j = 0; j < c->cols; ++j)
            xin[j] = oracle_bf16_to_f64(xr[j]);
        softmax_row_f64(xin, yout, c->cols);
        for (size_t j = 0; j < c->cols; ++j)
            yr[j] = oracle_round_to_bf16(yout[j]);
    }
    free(yout);
    free(xin);
}

/* double in, double out */
void oracle_softmax_rows_f64(const double *x, double *y, size_t rows, size_t cols, int nthreads)
{
    softmax_ctx c = {x, y, cols};
    parallel_ranges(softmax_f64_range, &c, rows, nthreads);
}

/* fp32 in, computed in double, rounded once to fp32 */
void oracle_softmax_rows_f32(const float *x, float *y, size_t rows, size_t cols, int nthreads)
{
    softmax_ctx c = {x, y, cols};
    parallel_ranges(softmax_f32_range, &c, rows, nthreads);
}

/* bf16 (raw 16-bit patterns) in, computed in double, rounded once to bf16 */
void oracle_softmax_rows_bf16(const uint16_t *x, uint16_t *y, size_t rows, size_t cols, int nthreads)
{
    softmax_ctx c = {x, y, cols};
    parallel_ranges(softmax_bf16_range, &c, rows, nthreads);
}

/* ------------------------------------------------------------------ */
/* Scaled, causally masked row softmax                                  */
/* ------------------------------------------------------------------ */

/* The score step of causal attention (lecture 6, "GPU Kernels and Triton",
 * section 8): scores are scaled (by 1/sqrt(d_k) there), a score whose key
 * position is after its query position is replaced by -inf, and softmax is
 * taken over the row.  Here row r of a [rows, cols] matrix has query
 * position q = (r mod period) + offset and column j is key position j, so
 *     s_j = scale * x_j  for j <= q,   s_j = -inf  for j > q,
 * and y = softmax(s) as softmax_row_f64 defines it; period == 0 means no
 * mask.  Element kinds: 0 = double, 1 = fp32, 2 = bf16 patterns; outputs
 * are of the input's kind, rounded once from double. */
typedef struct {
    const void *x;
    void *y;
    int kind;
    size_t cols;
    double scale;
    size_t period, offset;
} causal_ctx;

static double causal_in(const causal_ctx *c, size_t i)
{
    if (c->kind == 0)
        return ((const double *)c->x)[i];
    if (c->kind == 1)
        return (double)((const float *)c->x)[i];
    return oracle_bf16_to_f64(((const uint16_t *)c->x)[i]);
}

static void causal_out(const causal_ctx *c, size_t i, double v)
{
    if (c->kind == 0)
        ((double *)c->y)[i] = v;
    else if (c->kind == 1)
        ((float *)c->y)[i] = oracle_round_to_f32(v);
    else
        ((uint16_t *)c->y)[i] = oracle_round_to_bf16(v);
}

static void softmax_causal_range(void *p, size_t b, size_t e)
{
    causal_ctx *c = (causal_ctx *)p;
    double *s = (double *)malloc(c->cols * sizeof(double) + 1);
    double *out = (double *)malloc(c->cols * sizeof(double) + 1);
    for (size_t r = b; r < e; ++r) {
        for (size_t j = 0; j < c->cols; ++j) {
            const int masked = c->period != 0 && j > (r % c->period) + c->offset;
            s[j] = masked ? -INFINITY : c->scale * causal_in(c, r * c->cols + j);
        }
        softmax_row_f64(s, out, c->cols);
        for (size_t j = 0; j < c->cols; ++j)
            causal_out(c, r * c->cols + j, out[j]);
    }
    free(out);
    free(s);
}

void oracle_softmax_rows_causal(const void *x, void *y, int kind, size_t rows, size_t cols, double scale,
                                size_t period, size_t offset, int nthreads)
{
    causal_ctx c = {x, y, kind, cols, scale, period, offset};
    parallel_ranges(softmax_causal_range, &c, rows, nthreads);
}

/* ------------------------------------------------------------------ */
/* LayerNorm over rows (+ optional GELU)                                */
/* ------------------------------------------------------------------ */

/* The normalisation step of the fused LayerNorm -> Linear -> GELU example
 * (lecture 6, "GPU Kernels and Triton", sections 6.1 and 6.2, where it is
 * F.layer_norm(x, x.shape[-1:])): over each row of a [rows, cols] matrix,
 *     mean = sum_j x_j / cols,   var = sum_j (x_j - mean)^2 / cols,
 *     y_j  = (x_j - mean) / sqrt(var + eps),
 * then y_j * gamma_j + beta_j when gamma / beta are given (either may be
 * NULL: 1 / 0), then GELU when asked (1 = tanh form, 2 = exact form) -- the
 * activation the same example applies.  Both sums are Neumaier-compensated;
 * the variance is taken about the computed mean (two passes). */
static void neumaier_add(double *s, double *c, double v)
{
    const double t = *s + v;
    if (fabs(*s) >= fabs(v))
        *c += (*s - t) + v;
    else
        *c += (v - t) + *s;
    *s = t;
}

typedef struct {
    const void *x;
    void *y;
    int kind; /* element kind as causal_ctx: 0 double, 1 fp32, 2 bf16 */
    size_t cols;
    const double *gamma, *beta;
    double eps;
    int gelu;
} layernorm_ctx;

static void layernorm_range(void *p, size_t b, size_t e)
{
    layernorm_ctx *c = (layernorm_ctx *)p;
    causal_ctx io = {c->x, c->y, c->kind, c->cols, 1.0, 0, 0};
    double *v = (double *)malloc(c->cols * sizeof(double) + 1);
    for (size_t r = b; r < e; ++r) {
        const size_t base = r * c->cols;
        double s = 0.0, comp = 0.0;
        for (size_t j = 0; j < c->cols; ++j) {
            v[j] = causal_in(&io, base + j);
            neumaier_add(&s, &comp, v[j]);
        }
        const double mean = (s + comp) / (double)c->cols;
        double q = 0.0, qc = 0.0;
        for (size_t j = 0; j < c->cols; ++j)
            neumaier_add(&q, &qc, (v[j] - mean) * (v[j] - mean));
        const double var = (q + qc) / (double)c->cols;
        const double rstd = 1.0 / sqrt(var + c->eps);
        for (size_t j = 0; j < c->cols; ++j) {
            double y = (v[j] - mean) * rstd;
            if (c->gamma)
                y *= c->gamma[j];
            if (c->beta)
                y += c->beta[j];
            if (c->gelu == 1)
                y = oracle_gelu_tanh(y);
            else if (c->gelu == 2)
                y = oracle_gelu_erf(y);
            causal_out(&io, base + j, y);
        }
    }
    free(v);
}

void oracle_layernorm_rows(const void *x, void *y, int kind, size_t rows, size_t cols, const double *gamma,
                           const double *beta, double eps, int gelu, int nthreads)
{
    layernorm_ctx c = {x, y, kind, cols, gamma, beta, eps, gelu};
    parallel_ranges(layernorm_range, &c, rows, nthreads);
}

/* ------------------------------------------------------------------ */
/* Attention forward                                                    */
/* ------------------------------------------------------------------ */

/* The attention that Flash Attention computes (lecture 6, "GPU Kernels and
 * Triton", sections 7.3 and 8): for each of `bh` independent (batch, head)
 * slices, with Q [tq, d], K [tk, d], V [tk, d] row-major,
 *     S = scale * Q K^T,
 *     S[i, j] = -inf where the key comes after the query (causal: query i
 *               sits at position i + (tk - tq) of the key sequence),
 *     P = softmax over each row of S (softmax_row_f64),
 *     O = P V.
 * Plain loops in double, no blocking; kinds as causal_ctx (0 double,
 * 1 fp32, 2 bf16 patterns) for Q, K, V and O alike, O rounded once. */
typedef struct {
    const void *q, *k, *v;
    void *o;
    int kind;
    size_t tq, tk, d;
    double scale;
    int causal;
} attn_ctx;

static double attn_in(const void *p, int kind, size_t i)
{
    causal_ctx io = {p, NULL, kind, 0, 1.0, 0, 0};
    return causal_in(&io, i);
}

static void attention_range(void *p, size_t b, size_t e)
{
    attn_ctx *c = (attn_ctx *)p;
    double *s = (double *)malloc(c->tk * sizeof(double) + 1);
    double *pr = (double *)malloc(c->tk * sizeof(double) + 1);
    causal_ctx out = {NULL, c->o, c->kind, 0, 1.0, 0, 0};
    /* one (slice, query) pair per unit of work */
    for (size_t u = b; u < e; ++u) {
        const size_t h = u / c->tq, i = u % c->tq;
        const size_t qb = (h * c->tq + i) * c->d;
        for (size_t j = 0; j < c->tk; ++j) {
            if (c->causal && j > i + (c->tk - c->tq)) {
                s[j] = -INFINITY;
                continue;
            }
            const size_t kb = (h * c->tk + j) * c->d;
            double dot = 0.0;
            for (size_t t = 0; t < c->d; ++t)
                dot += attn_in(c->q, c->kind, qb + t) * attn_in(c->k, c->kind, kb + t);
            s[j] = c->scale * dot;
        }
        softmax_row_f64(s, pr, c->tk);
        for (size_t t = 0; t < c->d; ++t) {
            double acc = 0.0;
            for (size_t j = 0; j < c->tk; ++j)
                if (pr[j] != 0.0)
                    acc += pr[j] * attn_in(c->v, c->kind, (h * c->tk + j) * c->d + t);
            causal_out(&out, qb + t, acc);
        }
    }
    free(pr);
    free(s);
}

void oracle_attention(const void *q, const void *k, const void *v, void *o, int kind, size_t bh, size_t tq,
                      size_t tk, size_t d, double scale, int causal, int nthreads)
{
    attn_ctx c = {q, k, v, o, kind, tq, tk, d, scale, causal};
    parallel_ranges(attention_range, &c, bh * tq, nthreads);
}

/* array forms of the rounding helpers */
void oracle_round_to_f32_array(const double *v, float *out, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_round_to_f32(v[i]);
}

void oracle_round_to_bf16_array(const double *v, uint16_t *out, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_round_to_bf16(v[i]);
}

void oracle_bf16_to_f64_array(const uint16_t *b, double *out, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_to_f64(b[i]);
}
