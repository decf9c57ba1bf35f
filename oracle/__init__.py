"""CPU oracle for tanh-GELU and row softmax (double precision).

TEST INFRASTRUCTURE ONLY.  This package is the independent checker for the
CUDA library in ``memory_bound_fk_b200``; it shares no code with it and
neither imports the other.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

The arithmetic lives in ``fk_oracle.c`` (plain C, IEEE double, no blocking or
reordering); this module only marshals numpy arrays into it.

Definitions followed:
  * GELU (tanh form): lecture-6 notes of CS336 (kyc001.github.io), section 4.2,
    0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
  * GELU (exact form): x Phi(x), the function the tanh form approximates
    (the lecture's fusion example, section 6, calls PyTorch's default gelu).
  * Row softmax: "Lecture 6: GPU Kernels and Triton" (cs336.sjfarmltd.com),
    section 7.2 (standard two-pass form), and the lecture-6 notes, section 5.2
    (row max, then exponentials and their sum, then normalise).
  * Scaled, causally masked softmax: the same lecture, section 8 (scores
    scaled, -inf where the key comes after the query, then softmax).
  * LayerNorm (+ GELU): the same lecture, sections 6.1-6.2 (the fused
    LayerNorm -> Linear -> GELU example; F.layer_norm over the last axis).
  * Attention forward: the same lecture, sections 7.3 and 8 (what Flash
    Attention computes: softmax(scale Q K^T, causal mask) V).

Parity pins: every function here is pinned by tests in
``tests/test_oracle_pins.py`` (closed forms, invariants, library routines
of the same definition, brute force on tiny inputs).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        d, f, u16 = ctypes.c_double, ctypes.c_float, ctypes.c_uint16
        p, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        lib.oracle_gelu_tanh.argtypes = [d]
        lib.oracle_gelu_tanh.restype = d
        lib.oracle_round_to_f32.argtypes = [d]
        lib.oracle_round_to_f32.restype = f
        lib.oracle_round_to_bf16.argtypes = [d]
        lib.oracle_round_to_bf16.restype = u16
        lib.oracle_bf16_to_f64.argtypes = [u16]
        lib.oracle_bf16_to_f64.restype = d
        lib.oracle_gelu_erf.argtypes = [d]
        lib.oracle_gelu_erf.restype = d
        for name in ("oracle_gelu_tanh_f64", "oracle_gelu_tanh_f32", "oracle_gelu_erf_f64"):
            getattr(lib, name).argtypes = [p, p, sz, i]
            getattr(lib, name).restype = None
        for name in ("oracle_softmax_rows_f64", "oracle_softmax_rows_f32",
                     "oracle_softmax_rows_bf16"):
            getattr(lib, name).argtypes = [p, p, sz, sz, i]
            getattr(lib, name).restype = None
        lib.oracle_softmax_rows_causal.argtypes = [p, p, i, sz, sz, d, sz, sz, i]
        lib.oracle_softmax_rows_causal.restype = None
        lib.oracle_layernorm_rows.argtypes = [p, p, i, sz, sz, p, p, d, i, i]
        lib.oracle_layernorm_rows.restype = None
        lib.oracle_attention.argtypes = [p, p, p, p, i, sz, sz, sz, sz, d, i, i]
        lib.oracle_attention.restype = None
        for name in ("oracle_round_to_f32_array", "oracle_round_to_bf16_array",
                     "oracle_bf16_to_f64_array"):
            getattr(lib, name).argtypes = [p, p, sz]
            getattr(lib, name).restype = None
        _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---------------------------------------------------------------- scalars

def gelu_tanh(x: float) -> float:
    """GELU (tanh form) of one double."""
    return _load().oracle_gelu_tanh(float(x))


def round_to_f32_scalar(v: float) -> np.float32:
    return np.float32(_load().oracle_round_to_f32(float(v)))


def round_to_bf16_scalar(v: float) -> int:
    return int(_load().oracle_round_to_bf16(float(v)))


# ---------------------------------------------------------------- arrays

def gelu_tanh_f64(x: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """Elementwise GELU (tanh form), double in, double out."""
    x = _c(x, np.float64)
    y = np.empty_like(x)
    _load().oracle_gelu_tanh_f64(_ptr(x), _ptr(y), x.size, nthreads or default_threads())
    return y


def gelu_erf(x: float) -> float:
    """Exact GELU, x * Phi(x), of one double."""
    return _load().oracle_gelu_erf(float(x))


def gelu_erf_f64(x: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """Elementwise exact GELU, double in, double out."""
    x = _c(x, np.float64)
    y = np.empty_like(x)
    _load().oracle_gelu_erf_f64(_ptr(x), _ptr(y), x.size, nthreads or default_threads())
    return y


def gelu_tanh_f32(x: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """fp32 in; computed in double; rounded once to fp32 (nearest even)."""
    x = _c(x, np.float32)
    y = np.empty_like(x)
    _load().oracle_gelu_tanh_f32(_ptr(x), _ptr(y), x.size, nthreads or default_threads())
    return y


def _rows_cols(x: np.ndarray):
    if x.ndim != 2:
        raise ValueError("softmax oracle expects a 2-D [rows, cols] array")
    return x.shape


def softmax_rows_f64(x: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """Softmax over the last axis of a [rows, cols] matrix, double in/out."""
    x = _c(x, np.float64)
    rows, cols = _rows_cols(x)
    y = np.empty_like(x)
    _load().oracle_softmax_rows_f64(_ptr(x), _ptr(y), rows, cols, nthreads or default_threads())
    return y


def softmax_rows_f32(x: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """fp32 rows in; computed in double; rounded once to fp32."""
    x = _c(x, np.float32)
    rows, cols = _rows_cols(x)
    y = np.empty_like(x)
    _load().oracle_softmax_rows_f32(_ptr(x), _ptr(y), rows, cols, nthreads or default_threads())
    return y


def softmax_rows_bf16(x_bits: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """bf16 rows given as uint16 bit patterns; computed in double; rounded
    once to bf16 (nearest even).  Returns uint16 bit patterns."""
    x = _c(x_bits, np.uint16)
    rows, cols = _rows_cols(x)
    y = np.empty_like(x)
    _load().oracle_softmax_rows_bf16(_ptr(x), _ptr(y), rows, cols, nthreads or default_threads())
    return y


def softmax_rows_causal(x: np.ndarray, scale: float, period: int, offset: int = 0,
                        nthreads: int | None = None) -> np.ndarray:
    """Scaled, causally masked row softmax of a [rows, cols] matrix: row r
    keeps columns j <= (r mod period) + offset (all when period == 0), scores
    scale * x_j, -inf elsewhere, then softmax.  float64 in -> float64 out;
    float32 in -> float32 out; uint16 (bf16 patterns) in -> uint16 out, each
    computed in double and rounded once."""
    if x.dtype == np.float64:
        kind = 0
    elif x.dtype == np.float32:
        kind = 1
    elif x.dtype == np.uint16:
        kind = 2
    else:
        raise TypeError("float64, float32 or uint16 (bf16 bits)")
    x = np.ascontiguousarray(x)
    rows, cols = _rows_cols(x)
    if period < 0 or offset < 0:
        raise ValueError("period and offset are non-negative")
    y = np.empty_like(x)
    _load().oracle_softmax_rows_causal(_ptr(x), _ptr(y), kind, rows, cols, float(scale), int(period), int(offset),
                                       nthreads or default_threads())
    return y


_GELU_CODES = {None: 0, "tanh": 1, "erf": 2}


def layernorm_rows(x: np.ndarray, eps: float = 1e-5, gamma=None, beta=None, gelu: str | None = None,
                   nthreads: int | None = None) -> np.ndarray:
    """LayerNorm over the last axis of a [rows, cols] matrix (mean and biased
    variance of each row, (x - mean) / sqrt(var + eps)), then * gamma + beta
    (each optional, length cols), then GELU ("tanh", "erf" or None).  float64
    in -> float64 out; float32 -> float32; uint16 (bf16 patterns) -> uint16;
    computed in double and rounded once."""
    kinds = {np.dtype(np.float64): 0, np.dtype(np.float32): 1, np.dtype(np.uint16): 2}
    if x.dtype not in kinds:
        raise TypeError("float64, float32 or uint16 (bf16 bits)")
    x = np.ascontiguousarray(x)
    rows, cols = _rows_cols(x)
    g = None if gamma is None else _c(gamma, np.float64)
    b = None if beta is None else _c(beta, np.float64)
    for a in (g, b):
        if a is not None and a.shape != (cols,):
            raise ValueError("gamma / beta must have cols elements")
    y = np.empty_like(x)
    _load().oracle_layernorm_rows(_ptr(x), _ptr(y), kinds[x.dtype], rows, cols,
                                  None if g is None else _ptr(g), None if b is None else _ptr(b),
                                  float(eps), _GELU_CODES[gelu], nthreads or default_threads())
    return y


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, causal: bool,
              nthreads: int | None = None) -> np.ndarray:
    """Attention forward over [bh, t, d] arrays (q: [bh, tq, d]; k, v:
    [bh, tk, d]): softmax(scale * q k^T, causal mask with query i at key
    position i + tk - tq) v.  float64 in -> float64 out; float32 -> float32;
    uint16 (bf16 patterns) -> uint16; computed in double, rounded once."""
    kinds = {np.dtype(np.float64): 0, np.dtype(np.float32): 1, np.dtype(np.uint16): 2}
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in kinds:
        raise TypeError("q, k, v: one of float64, float32, uint16 (bf16 bits)")
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    if q.ndim != 3 or k.shape != v.shape or k.ndim != 3 or q.shape[0] != k.shape[0] or q.shape[2] != k.shape[2]:
        raise ValueError("shapes [bh, tq, d], [bh, tk, d], [bh, tk, d]")
    bh, tq, d = q.shape
    tk = k.shape[1]
    if causal and tk < tq:
        raise ValueError("causal attention needs tk >= tq")
    o = np.empty_like(q)
    _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), kinds[q.dtype], bh, tq, tk, d, float(scale),
                             int(bool(causal)), nthreads or default_threads())
    return o


def round_to_f32(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.float32)
    _load().oracle_round_to_f32_array(_ptr(v), _ptr(out), v.size)
    return out


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """double -> bf16 bit patterns (uint16), one rounding, nearest even."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_round_to_bf16_array(_ptr(v), _ptr(out), v.size)
    return out


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact double values."""
    b = _c(b, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().oracle_bf16_to_f64_array(_ptr(b), _ptr(out), b.size)
    return out


__all__ = [
    "gelu_tanh", "gelu_tanh_f64", "gelu_tanh_f32", "gelu_erf", "gelu_erf_f64",
    "softmax_rows_f64", "softmax_rows_f32", "softmax_rows_bf16", "softmax_rows_causal", "layernorm_rows", "attention",
    "round_to_f32", "round_to_bf16", "round_to_f32_scalar", "round_to_bf16_scalar",
    "bf16_to_f64", "default_threads",
]
