"""Seeded synthetic inputs for the GELU and row-softmax workloads.

This module only draws random numbers and lays them out; it holds none of
the operators' arithmetic.  It is the one piece shared by the CUDA-side
callers (bench, tests) and the CPU oracle's callers, so that both see
bit-identical inputs.

Random source: numpy's PCG64.  Large inputs are generated in fixed chunks,
each with its own generator derived from ``SeedSequence(seed,
spawn_key=(chunk,))``, so the bits do not depend on how many host threads
generate them (numpy releases the GIL while filling arrays).

Workloads (shapes, distributions and structure of the lecture pages'
workloads; every value is synthetic):

=============  ==============================================================
cfg1_softmax   fp32 [256, 1000], i.i.d. N(0, 3^2), seed 0
cfg1_gelu      fp32 [256000], the same values as cfg1_softmax
cfg2_gelu      fp32 [8388608] (32 MiB), N(0, 1); exactly round(0.01 n) = 83886
               positions, chosen without replacement, redrawn U[-20, 20]; seed 1
cfg3_softmax   fp32 [8192, 4096], N(0, 4^2); in every row exactly 410
               (= round(0.1 * 4096)) positions, chosen without replacement, set
               to -inf; seed 2
cfg4_softmax   bf16 [1048576, 2048] = 32 x 16 heads of 2048 x 2048 attention
               scores, N(0, 8^2) rounded to bf16 (nearest even); causal mask:
               column j > (row mod 2048) is -inf; seed 3
cfg5_softmax   fp32 [512, 131072] (256 MiB), N(0, 2^2), plus 50 added at one
               uniformly drawn position per row; seed 4
=============  ==============================================================

bf16 arrays are returned as ``uint16`` bit patterns.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

NEG_INF_BF16 = np.uint16(0xFF80)


@dataclass(frozen=True)
class Workload:
    name: str
    op: str          # "gelu" or "softmax"
    dtype: str       # "f32" or "bf16"
    shape: tuple     # (n,) for gelu, (rows, cols) for softmax
    seed: int
    recipe: str

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n

    @property
    def itemsize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def algorithmic_bytes(self) -> int:
        return algorithmic_bytes(self.op, self.itemsize, self.shape)


def algorithmic_bytes(op: str, itemsize: int, shape: tuple) -> int:
    """One read of the input plus one write of the output.  For the causal
    softmax (rows in blocks of T = cols queries against T keys) only the kept
    entries are read: row i of a block reads i + 1 of its T values; with
    masked stores skipped, only those are written too."""
    if op in ("attention", "attention_full"):
        _, bh, t, d = shape
        return 4 * bh * t * d * itemsize  # q, k, v read, o written
    if op in ("softmax_causal", "softmax_causal_skip"):
        rows, cols = shape
        full, rem = divmod(rows, cols)
        kept = full * cols * (cols + 1) // 2 + rem * (rem + 1) // 2
        return (kept + (kept if op == "softmax_causal_skip" else rows * cols)) * itemsize
    n = 1
    for d in shape:
        n *= d
    return 2 * n * itemsize


WORKLOADS = {
    w.name: w for w in [
        Workload("cfg1_softmax", "softmax", "f32", (256, 1000), 0,
                 "fp32 256x1000, iid N(0,3^2), seed 0"),
        Workload("cfg1_gelu", "gelu", "f32", (256000,), 0,
                 "fp32 256000, the cfg1_softmax values"),
        Workload("cfg2_gelu", "gelu", "f32", (8388608,), 1,
                 "fp32 8388608, N(0,1) with 83886 positions redrawn U[-20,20]"),
        Workload("cfg3_softmax", "softmax", "f32", (8192, 4096), 2,
                 "fp32 8192x4096, N(0,4^2), 410 -inf per row"),
        Workload("cfg4_softmax", "softmax", "bf16", (32 * 16 * 2048, 2048), 3,
                 "bf16 1048576x2048 (32x16 heads x 2048 queries), N(0,8^2), causal -inf"),
        Workload("cfg5_softmax", "softmax", "f32", (512, 131072), 4,
                 "fp32 512x131072, N(0,2^2), +50 at one position per row"),
        # variants of the same operators (exact GELU, bf16 GELU, softmax with
        # the causal mask generated in the kernel)
        Workload("cfg2_gelu_erf", "gelu_erf", "f32", (8388608,), 1,
                 "the cfg2_gelu values, exact GELU x*Phi(x)"),
        Workload("gelu_bf16", "gelu", "bf16", (16777216,), 5,
                 "bf16 16777216 (32 MiB), N(0,1) with 167772 positions redrawn U[-20,20]"),
        Workload("gelu_erf_bf16", "gelu_erf", "bf16", (16777216,), 5,
                 "the gelu_bf16 values, exact GELU x*Phi(x)"),
        Workload("cfg4_causal", "softmax_causal", "bf16", (32 * 16 * 2048, 2048), 3,
                 "the cfg4_softmax scores, causal mask generated in the kernel (masked entries not read)"),
        Workload("cfg4_causal_skip", "softmax_causal_skip", "bf16", (32 * 16 * 2048, 2048), 3,
                 "as cfg4_causal, masked outputs not stored either (FK_SOFTMAX_SKIP_MASKED)"),
        # LayerNorm over transformer-shaped activations (hidden size 4096)
        Workload("ln_f32", "layernorm", "f32", (16384, 4096), 6,
                 "fp32 16384x4096, row r ~ N(mu_r, s_r^2), mu_r ~ U[-2,2], s_r ~ U[0.5,2]; "
                 "gamma ~ 1+N(0,0.1^2), beta ~ N(0,0.1^2); eps 1e-5"),
        Workload("ln_gelu_bf16", "layernorm_gelu", "bf16", (65536, 4096), 7,
                 "bf16 65536x4096, same recipe, then tanh-GELU"),
        # attention forward: q, k, v stacked as [3, batch*heads, t, d]
        Workload("attn_causal_bf16", "attention", "bf16", (3, 4 * 16, 2048, 128), 8,
                 "q, k, v: 4 x 16 heads x 2048 x 128 bf16, N(0,1); causal; scale 1/sqrt(128)"),
        Workload("attn_bf16", "attention_full", "bf16", (3, 4 * 16, 2048, 128), 9,
                 "as attn_causal_bf16 without the mask"),
    ]
}


def _threads(threads: int | None) -> int:
    if threads:
        return threads
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def chunk_rng(seed: int, chunk: int) -> np.random.Generator:
    """Independent generator for one chunk of a workload."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(chunk,))))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Pack fp32 values into bf16 bit patterns, round to nearest even.
    (Input preparation only; finite inputs.)"""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ------------------------------------------------------------------ cfg 1

def _cfg1_values() -> np.ndarray:
    g = np.random.default_rng(0)
    return (g.standard_normal(256000) * 3.0).astype(np.float32)


# ------------------------------------------------------------------ cfg 2

def _cfg2(n: int = 8388608, seed: int = 1) -> np.ndarray:
    g = np.random.default_rng(seed)
    x = g.standard_normal(n, dtype=np.float32)
    k = int(round(0.01 * n))
    pos = g.choice(n, size=k, replace=False)
    x[pos] = g.uniform(-20.0, 20.0, size=k).astype(np.float32)
    return x


# ------------------------------------------------------------------ cfg 3

CFG3_ROWS_PER_CHUNK = 64


def _cfg3_chunk(out: np.ndarray, chunk: int, seed: int, n_inf: int) -> None:
    rows, cols = out.shape
    g = chunk_rng(seed, chunk)
    g.standard_normal(out=out, dtype=np.float32)
    out *= np.float32(4.0)
    for r in range(rows):
        out[r, g.choice(cols, size=n_inf, replace=False)] = -np.inf


def cfg3_rows(row_begin: int, row_end: int, cols: int = 4096, seed: int = 2) -> np.ndarray:
    """Rows [row_begin, row_end) of cfg3 (chunk-aligned generation)."""
    n_inf = int(round(0.1 * cols))
    c0, c1 = row_begin // CFG3_ROWS_PER_CHUNK, (row_end - 1) // CFG3_ROWS_PER_CHUNK + 1
    buf = np.empty(((c1 - c0) * CFG3_ROWS_PER_CHUNK, cols), np.float32)
    for c in range(c0, c1):
        _cfg3_chunk(buf[(c - c0) * CFG3_ROWS_PER_CHUNK:(c - c0 + 1) * CFG3_ROWS_PER_CHUNK], c, seed, n_inf)
    off = c0 * CFG3_ROWS_PER_CHUNK
    return buf[row_begin - off:row_end - off].copy()


def _cfg3(rows: int = 8192, cols: int = 4096, seed: int = 2, threads=None) -> np.ndarray:
    assert rows % CFG3_ROWS_PER_CHUNK == 0
    n_inf = int(round(0.1 * cols))
    x = np.empty((rows, cols), np.float32)
    nchunks = rows // CFG3_ROWS_PER_CHUNK
    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(lambda c: _cfg3_chunk(
            x[c * CFG3_ROWS_PER_CHUNK:(c + 1) * CFG3_ROWS_PER_CHUNK], c, seed, n_inf), range(nchunks)))
    return x


# ------------------------------------------------------------------ cfg 4

CFG4_T = 2048          # queries per head = keys per head
CFG4_HEADS = 32 * 16   # batch x heads


def _cfg4_head(out: np.ndarray, head: int, seed: int) -> None:
    """One head: out is the uint16 [T, T] block of that head."""
    t = out.shape[0]
    g = chunk_rng(seed, head)
    s = g.standard_normal((t, t), dtype=np.float32)
    s *= np.float32(8.0)
    out[...] = f32_to_bf16_bits(s)
    for i in range(t - 1):                      # key j > query i is masked
        out[i, i + 1:] = NEG_INF_BF16


def cfg4_head(head: int, seed: int = 3, t: int = CFG4_T) -> np.ndarray:
    out = np.empty((t, t), np.uint16)
    _cfg4_head(out, head, seed)
    return out


def _cfg4(heads: int = CFG4_HEADS, t: int = CFG4_T, seed: int = 3, threads=None) -> np.ndarray:
    x = np.empty((heads * t, t), np.uint16)
    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(lambda h: _cfg4_head(x[h * t:(h + 1) * t], h, seed), range(heads)))
    return x


# ------------------------------------------------------------------ cfg 5

CFG5_ROWS_PER_CHUNK = 8


def _cfg5_chunk(out: np.ndarray, chunk: int, seed: int) -> None:
    rows, cols = out.shape
    g = chunk_rng(seed, chunk)
    g.standard_normal(out=out, dtype=np.float32)
    out *= np.float32(2.0)
    pos = g.integers(0, cols, size=rows)
    out[np.arange(rows), pos] += np.float32(50.0)


def cfg5_rows(row_begin: int, row_end: int, cols: int = 131072, seed: int = 4) -> np.ndarray:
    c0, c1 = row_begin // CFG5_ROWS_PER_CHUNK, (row_end - 1) // CFG5_ROWS_PER_CHUNK + 1
    buf = np.empty(((c1 - c0) * CFG5_ROWS_PER_CHUNK, cols), np.float32)
    for c in range(c0, c1):
        _cfg5_chunk(buf[(c - c0) * CFG5_ROWS_PER_CHUNK:(c - c0 + 1) * CFG5_ROWS_PER_CHUNK], c, seed)
    off = c0 * CFG5_ROWS_PER_CHUNK
    return buf[row_begin - off:row_end - off].copy()


def _cfg5(rows: int = 512, cols: int = 131072, seed: int = 4, threads=None) -> np.ndarray:
    assert rows % CFG5_ROWS_PER_CHUNK == 0
    x = np.empty((rows, cols), np.float32)
    nchunks = rows // CFG5_ROWS_PER_CHUNK
    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(lambda c: _cfg5_chunk(
            x[c * CFG5_ROWS_PER_CHUNK:(c + 1) * CFG5_ROWS_PER_CHUNK], c, seed), range(nchunks)))
    return x


# ------------------------------------------------------------------ public

def make(name: str, threads: int | None = None, rows: int | None = None) -> np.ndarray:
    """Input of a named workload (fp32 array, or uint16 bf16 bits).

    `rows` (softmax) or element count (GELU) shrinks the workload to its
    leading part with the same recipe -- for small profiling cases; None is
    the full size."""
    if name == "cfg1_softmax":
        return _cfg1_values().reshape(256, 1000)[:rows]
    if name == "cfg1_gelu":
        return _cfg1_values()[:rows]
    if name == "cfg2_gelu":
        return _cfg2()[:rows]
    if name == "cfg3_softmax":
        r = rows or 8192
        return _cfg3(rows=-(-r // CFG3_ROWS_PER_CHUNK) * CFG3_ROWS_PER_CHUNK, threads=threads)[:r]
    if name in ("cfg4_softmax", "cfg4_causal", "cfg4_causal_skip"):
        r = rows or CFG4_HEADS * CFG4_T
        return _cfg4(heads=-(-r // CFG4_T), threads=threads)[:r]
    if name == "cfg2_gelu_erf":
        return _cfg2()[:rows]
    if name in ("gelu_bf16", "gelu_erf_bf16"):
        return f32_to_bf16_bits(_cfg2(16777216, seed=5))[:rows]
    if name in ("attn_causal_bf16", "attn_bf16"):
        w = WORKLOADS[name]
        shape = w.shape if rows is None else (3, rows, w.shape[2], w.shape[3])
        return f32_to_bf16_bits(np.random.default_rng(w.seed).standard_normal(shape, dtype=np.float32))
    if name in ("ln_f32", "ln_gelu_bf16"):
        w = WORKLOADS[name]
        r = rows or w.shape[0]
        return layernorm_input(r, w.shape[1], w.dtype, w.seed, threads=threads)
    if name == "cfg5_softmax":
        r = rows or 512
        return _cfg5(rows=-(-r // CFG5_ROWS_PER_CHUNK) * CFG5_ROWS_PER_CHUNK, threads=threads)[:r]
    raise KeyError(name)


def normal(shape, sigma: float, seed: int, dtype: str = "f32") -> np.ndarray:
    """Generic i.i.d. N(0, sigma^2) test input (fp32, or bf16 bits)."""
    g = np.random.default_rng(seed)
    x = (g.standard_normal(shape) * sigma).astype(np.float32)
    return x if dtype == "f32" else f32_to_bf16_bits(x)


def causal_scores(heads: int, t: int, sigma: float, seed: int) -> np.ndarray:
    """Attention-score-shaped bf16 bits: heads x [t, t], causal -inf mask."""
    x = np.empty((heads * t, t), np.uint16)
    for h in range(heads):
        g = chunk_rng(seed, h)
        s = g.standard_normal((t, t), dtype=np.float32) * np.float32(sigma)
        b = f32_to_bf16_bits(s)
        for i in range(t - 1):
            b[i, i + 1:] = NEG_INF_BF16
        x[h * t:(h + 1) * t] = b
    return x


def softmax_input(rows: int, cols: int, dtype: str = "f32", sigma: float = 4.0,
                  neg_inf_frac: float = 0.0, seed: int = 0, shift: float = 0.0) -> np.ndarray:
    """Generic row-softmax test input: N(shift, sigma^2) entries, and in each
    row round(neg_inf_frac * cols) positions (without replacement) set to
    -inf.  fp32 array, or bf16 bits."""
    g = np.random.default_rng(seed)
    x = (g.standard_normal((rows, cols)) * sigma + shift).astype(np.float32)
    k = int(round(neg_inf_frac * cols))
    if k:
        for r in range(rows):
            x[r, g.choice(cols, size=k, replace=False)] = -np.inf
    if dtype == "f32":
        return x
    b = f32_to_bf16_bits(np.where(np.isneginf(x), 0.0, x))
    b[np.isneginf(x)] = NEG_INF_BF16
    return b


# ------------------------------------------------------------------ LayerNorm

LN_ROWS_PER_CHUNK = 256


def _ln_chunk(out: np.ndarray, chunk: int, seed: int) -> None:
    rows, cols = out.shape
    g = chunk_rng(seed, chunk)
    mu = g.uniform(-2.0, 2.0, size=(rows, 1)).astype(np.float32)
    sd = g.uniform(0.5, 2.0, size=(rows, 1)).astype(np.float32)
    g.standard_normal(out=out, dtype=np.float32)
    out *= sd
    out += mu


def layernorm_input(rows: int, cols: int, dtype: str = "f32", seed: int = 6, threads=None) -> np.ndarray:
    """LayerNorm activations: row r is N(mu_r, s_r^2) with mu_r ~ U[-2, 2]
    and s_r ~ U[0.5, 2], generated in chunks of 256 rows (fp32, or bf16
    bits)."""
    nchunks = -(-rows // LN_ROWS_PER_CHUNK)
    x = np.empty((nchunks * LN_ROWS_PER_CHUNK, cols), np.float32)
    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(lambda c: _ln_chunk(x[c * LN_ROWS_PER_CHUNK:(c + 1) * LN_ROWS_PER_CHUNK], c, seed),
                    range(nchunks)))
    x = x[:rows]
    return x if dtype == "f32" else f32_to_bf16_bits(x)


def layernorm_params(cols: int, seed: int = 6) -> tuple[np.ndarray, np.ndarray]:
    """gamma ~ 1 + N(0, 0.1^2) and beta ~ N(0, 0.1^2), fp32."""
    g = chunk_rng(seed, 1 << 30)
    gamma = (1.0 + 0.1 * g.standard_normal(cols)).astype(np.float32)
    beta = (0.1 * g.standard_normal(cols)).astype(np.float32)
    return gamma, beta


def attention_flops(bh: int, t: int, d: int, causal: bool) -> int:
    """Algorithmic FLOPs of attention forward: 2 d per (query, key) pair for
    q . k and 2 d for p v, over the unmasked pairs (t (t + 1) / 2 of t^2 per
    slice when causal)."""
    pairs = t * (t + 1) // 2 if causal else t * t
    return 4 * d * bh * pairs
