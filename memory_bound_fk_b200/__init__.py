"""memory_bound_fk_b200 -- fused memory-bound operators for NVIDIA B200 (sm_100a).

Python binding of ``libfk.so`` (declared in ``include/fk.h``).  This module
only marshals arguments: every step of the computation runs in the
library's CUDA kernels.  PyTorch provides device memory and streams.

Raw C-ABI mirrors (same names, pointers as integers, stream as a
``cudaStream_t`` integer):
    fk_gelu_tanh(x, y, n, stream) -> status
    fk_gelu(x, y, n, dtype, kind, stream) -> status
    fk_copy(src, dst, bytes, stream) -> status     (bandwidth reference)
    fk_softmax_rows(x, y, rows, cols, dtype, stream) -> status
    fk_softmax_rows_ex(x, y, rows, cols, dtype, plan, stream) -> status
    fk_softmax_rows_plan(rows, cols, dtype, path=FK_PATH_AUTO) -> SoftmaxPlan
    fk_softmax_rows_workspace(rows, cols, dtype, plan=None) -> bytes
    fk_softmax_rows_ws(x, y, rows, cols, dtype, plan, workspace, workspace_bytes, stream) -> status
    fk_softmax_rows_causal(x, y, rows, cols, dtype, scale, period, offset, stream) -> status
    fk_softmax_rows_causal_ex(x, y, rows, cols, dtype, scale, period, offset, flags, plan, stream) -> status
    fk_layernorm_rows(x, y, gamma, beta, rows, cols, dtype, eps, epilogue, stream) -> status
    fk_layernorm_rows_ex(x, y, gamma, beta, rows, cols, dtype, eps, epilogue, plan, stream) -> status
    fk_layernorm_rows_plan(rows, cols, dtype, path=FK_PATH_AUTO) -> SoftmaxPlan
    fk_attention_fwd(q, k, v, o, bh, t, d, causal, scale, stream) -> status
    fk_status_string(status) -> str
    fk_wait_timeouts(reset=False) -> int     (bounded-wait give-ups, synchronous)
    fk_wait_selftest(timeout_us, stream) -> status

Tensor conveniences (contiguous CUDA tensors; the current torch stream):
    gelu_tanh(x, out=None)
    gelu(x, out=None, approximate="tanh")   # fp32 / bf16; "tanh" or "none" (exact)
    softmax_rows(x, out=None, plan=None)    # softmax over the last dimension
    softmax_causal(x, scale, period=None, offset=0, out=None, plan=None)
    layernorm(x, eps=1e-5, weight=None, bias=None, gelu=None, out=None, plan=None)
    attention(q, k, v, causal=True, scale=None, out=None)   # [..., t, d] bf16

There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfk.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "fk.h")

# fk_status
FK_OK = 0
FK_ERR_INVALID_ARG = 1
FK_ERR_UNSUPPORTED_DTYPE = 2
FK_ERR_UNSUPPORTED_DEVICE = 3
FK_ERR_CUDA = 4
# fk_dtype
FK_F32 = 0
FK_BF16 = 1
# fk_gelu_kind
FK_GELU_TANH = 0
FK_GELU_ERF = 1
# fk_softmax_rows_causal_ex flags
FK_SOFTMAX_SKIP_MASKED = 1
# fk_epilogue
FK_EPILOGUE_NONE = 0
FK_EPILOGUE_GELU_TANH = 1
FK_EPILOGUE_GELU_ERF = 2
# fk_softmax_path
FK_PATH_AUTO = 0
FK_PATH_WARP = 1
FK_PATH_CTA = 2
FK_PATH_CLUSTER = 3
FK_PATH_TWOPHASE = 4
FK_PATH_SPLIT = 5
PATH_NAMES = {FK_PATH_WARP: "warp", FK_PATH_CTA: "cta", FK_PATH_CLUSTER: "cluster",
              FK_PATH_TWOPHASE: "twophase", FK_PATH_SPLIT: "split"}


class FkError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {fk_status_string(status)}"
                         + (f" (cudaError {fk_last_cuda_error()})" if status == FK_ERR_CUDA else ""))


class SoftmaxPlan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("threads", ctypes.c_int),
                ("vpt", ctypes.c_int), ("cluster", ctypes.c_int), ("chunks", ctypes.c_int)]

    def as_dict(self) -> dict:
        return {"path": PATH_NAMES.get(self.path, self.path), "threads": self.threads,
                "vpt": self.vpt, "cluster": self.cluster, "chunks": self.chunks}

    def __repr__(self) -> str:
        return f"SoftmaxPlan({self.as_dict()})"


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfk.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfk.so not found at {LIB_PATH}; build it with "
                              "`python -m memory_bound_fk_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, ci = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.fk_gelu_tanh.argtypes = [vp, vp, sz, vp]
        L.fk_gelu_tanh.restype = ci
        L.fk_copy.argtypes = [vp, vp, sz, vp]
        L.fk_copy.restype = ci
        L.fk_gelu.argtypes = [vp, vp, sz, ci, ci, vp]
        L.fk_gelu.restype = ci
        L.fk_softmax_rows.argtypes = [vp, vp, sz, sz, ci, vp]
        L.fk_softmax_rows.restype = ci
        L.fk_softmax_rows_ex.argtypes = [vp, vp, sz, sz, ci, ctypes.POINTER(SoftmaxPlan), vp]
        L.fk_softmax_rows_ex.restype = ci
        L.fk_softmax_rows_plan.argtypes = [sz, sz, ci, ci, ctypes.POINTER(SoftmaxPlan)]
        L.fk_softmax_rows_plan.restype = ci
        L.fk_status_string.argtypes = [ci]
        L.fk_status_string.restype = ctypes.c_char_p
        L.fk_last_cuda_error.argtypes = []
        L.fk_last_cuda_error.restype = ci
        L.fk_version.argtypes = []
        L.fk_version.restype = ci
        L.fk_softmax_rows_workspace.argtypes = [sz, sz, ci, ctypes.POINTER(SoftmaxPlan),
                                                ctypes.POINTER(ctypes.c_size_t)]
        L.fk_softmax_rows_workspace.restype = ci
        L.fk_softmax_rows_ws.argtypes = [vp, vp, sz, sz, ci, ctypes.POINTER(SoftmaxPlan), vp, sz, vp]
        L.fk_softmax_rows_ws.restype = ci
        L.fk_softmax_rows_causal.argtypes = [vp, vp, sz, sz, ci, ctypes.c_float, sz, sz, vp]
        L.fk_softmax_rows_causal.restype = ci
        L.fk_softmax_rows_causal_ex.argtypes = [vp, vp, sz, sz, ci, ctypes.c_float, sz, sz, ctypes.c_uint,
                                                ctypes.POINTER(SoftmaxPlan), vp]
        L.fk_softmax_rows_causal_ex.restype = ci
        L.fk_layernorm_rows.argtypes = [vp, vp, vp, vp, sz, sz, ci, ctypes.c_float, ci, vp]
        L.fk_layernorm_rows.restype = ci
        L.fk_layernorm_rows_ex.argtypes = [vp, vp, vp, vp, sz, sz, ci, ctypes.c_float, ci,
                                           ctypes.POINTER(SoftmaxPlan), vp]
        L.fk_layernorm_rows_ex.restype = ci
        L.fk_attention_fwd.argtypes = [vp, vp, vp, vp, sz, sz, sz, ci, ctypes.c_float, vp]
        L.fk_attention_fwd.restype = ci
        L.fk_layernorm_rows_plan.argtypes = [sz, sz, ci, ci, ctypes.POINTER(SoftmaxPlan)]
        L.fk_layernorm_rows_plan.restype = ci
        L.fk_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint), ci]
        L.fk_wait_timeouts.restype = ci
        L.fk_wait_selftest.argtypes = [ctypes.c_uint, vp]
        L.fk_wait_selftest.restype = ci
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the entry points declared in include/fk.h."""
    text = open(HEADER_PATH).read()
    return re.findall(r"FK_API\s+[\w\s\*]+?\b(fk_\w+)\s*\(", text)


# ---------------------------------------------------------------- raw mirrors

def fk_gelu_tanh(x: int, y: int, n: int, stream: int = 0) -> int:
    return lib().fk_gelu_tanh(x, y, n, stream)


def fk_copy(src: int, dst: int, nbytes: int, stream: int = 0) -> int:
    return lib().fk_copy(src, dst, nbytes, stream)


def fk_gelu(x: int, y: int, n: int, dtype: int, kind: int, stream: int = 0) -> int:
    return lib().fk_gelu(x, y, n, dtype, kind, stream)


def fk_softmax_rows(x: int, y: int, rows: int, cols: int, dtype: int, stream: int = 0) -> int:
    return lib().fk_softmax_rows(x, y, rows, cols, dtype, stream)


def fk_softmax_rows_ex(x: int, y: int, rows: int, cols: int, dtype: int,
                       plan: SoftmaxPlan | None, stream: int = 0) -> int:
    return lib().fk_softmax_rows_ex(x, y, rows, cols, dtype,
                                    ctypes.byref(plan) if plan is not None else None, stream)


def fk_softmax_rows_plan(rows: int, cols: int, dtype: int, path: int = FK_PATH_AUTO) -> SoftmaxPlan:
    p = SoftmaxPlan()
    st = lib().fk_softmax_rows_plan(rows, cols, dtype, path, ctypes.byref(p))
    if st != FK_OK:
        raise FkError(st, "fk_softmax_rows_plan")
    return p


def fk_softmax_rows_workspace(rows: int, cols: int, dtype: int, plan: SoftmaxPlan | None = None) -> int:
    """Workspace bytes a softmax call of this shape (and plan) needs."""
    b = ctypes.c_size_t(0)
    st = lib().fk_softmax_rows_workspace(rows, cols, dtype, ctypes.byref(plan) if plan is not None else None,
                                         ctypes.byref(b))
    if st != FK_OK:
        raise FkError(st, "fk_softmax_rows_workspace")
    return b.value


def fk_softmax_rows_ws(x: int, y: int, rows: int, cols: int, dtype: int, plan: SoftmaxPlan | None,
                       workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return lib().fk_softmax_rows_ws(x, y, rows, cols, dtype, ctypes.byref(plan) if plan is not None else None,
                                    workspace, workspace_bytes, stream)


def fk_softmax_rows_causal(x: int, y: int, rows: int, cols: int, dtype: int, scale: float, period: int,
                           offset: int = 0, stream: int = 0) -> int:
    return lib().fk_softmax_rows_causal(x, y, rows, cols, dtype, scale, period, offset, stream)


def fk_softmax_rows_causal_ex(x: int, y: int, rows: int, cols: int, dtype: int, scale: float, period: int,
                              offset: int, plan: SoftmaxPlan | None, stream: int = 0, flags: int = 0) -> int:
    return lib().fk_softmax_rows_causal_ex(x, y, rows, cols, dtype, scale, period, offset, flags,
                                           ctypes.byref(plan) if plan is not None else None, stream)


def fk_layernorm_rows(x: int, y: int, gamma: int, beta: int, rows: int, cols: int, dtype: int, eps: float,
                      epilogue: int = FK_EPILOGUE_NONE, stream: int = 0) -> int:
    return lib().fk_layernorm_rows(x, y, gamma or None, beta or None, rows, cols, dtype, eps, epilogue, stream)


def fk_layernorm_rows_ex(x: int, y: int, gamma: int, beta: int, rows: int, cols: int, dtype: int, eps: float,
                         epilogue: int, plan: SoftmaxPlan | None, stream: int = 0) -> int:
    return lib().fk_layernorm_rows_ex(x, y, gamma or None, beta or None, rows, cols, dtype, eps, epilogue,
                                      ctypes.byref(plan) if plan is not None else None, stream)


def fk_layernorm_rows_plan(rows: int, cols: int, dtype: int, path: int = FK_PATH_AUTO) -> SoftmaxPlan:
    p = SoftmaxPlan()
    st = lib().fk_layernorm_rows_plan(rows, cols, dtype, path, ctypes.byref(p))
    if st != FK_OK:
        raise FkError(st, "fk_layernorm_rows_plan")
    return p


def fk_attention_fwd(q: int, k: int, v: int, o: int, bh: int, t: int, d: int, causal: int, scale: float,
                     stream: int = 0) -> int:
    return lib().fk_attention_fwd(q, k, v, o, bh, t, d, causal, scale, stream)


def fk_status_string(status: int) -> str:
    return lib().fk_status_string(status).decode()


def fk_last_cuda_error() -> int:
    return lib().fk_last_cuda_error()


def fk_version() -> int:
    return lib().fk_version()


def fk_wait_timeouts(reset: bool = False) -> int:
    """Threads whose bounded cluster wait gave up on the current device
    (synchronous).  Raises FkError on failure."""
    c = ctypes.c_uint(0)
    st = lib().fk_wait_timeouts(ctypes.byref(c), 1 if reset else 0)
    if st != FK_OK:
        raise FkError(st, "fk_wait_timeouts")
    return c.value


def fk_wait_selftest(timeout_us: int, stream: int = 0) -> int:
    return lib().fk_wait_selftest(timeout_us, stream)


def fk_softmax_rows_noalloc(x: int, y: int, rows: int, cols: int, dtype: int, stream: int = 0) -> int:
    """fk_softmax_rows that never allocates device memory (scratch is a fixed
    1 MiB array inside the library; see include/fk.h)."""
    f = lib().fk_softmax_rows_noalloc
    if f.argtypes is None:
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        f.argtypes = [vp, vp, sz, sz, ctypes.c_int, vp]
        f.restype = ctypes.c_int
    return f(x, y, rows, cols, dtype, stream)


def fk_softmax_rows_noalloc_cap(x: int, y: int, rows: int, cols: int, dtype: int, capacity_pairs: int,
                                stream: int = 0) -> int:
    """fk_softmax_rows_noalloc on the first capacity_pairs entries of the
    library's scratch array (more batches on smaller inputs)."""
    f = lib().fk_softmax_rows_noalloc_cap
    if f.argtypes is None:
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        f.argtypes = [vp, vp, sz, sz, ctypes.c_int, sz, vp]
        f.restype = ctypes.c_int
    return f(x, y, rows, cols, dtype, capacity_pairs, stream)


def make_plan(path: int, threads: int = 0, vpt: int = 0, cluster: int = 0, chunks: int = 0) -> SoftmaxPlan:
    return SoftmaxPlan(path, threads, vpt, cluster, chunks)


# ---------------------------------------------------------------- tensors

def _stream_handle(t) -> int:
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _check_tensor(t, name: str):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gelu_tanh(x, out=None):
    """tanh-GELU of a contiguous fp32 CUDA tensor (``out`` may be ``x``)."""
    import torch
    _check_tensor(x, "x")
    if x.dtype != torch.float32:
        raise TypeError("gelu_tanh takes float32")
    if out is None:
        out = torch.empty_like(x)
    _check_tensor(out, "out")
    if out.dtype != x.dtype or out.numel() != x.numel() or out.device != x.device:
        raise ValueError("out must match x in dtype, size and device")
    st = fk_gelu_tanh(x.data_ptr(), out.data_ptr(), x.numel(), _stream_handle(x))
    if st != FK_OK:
        raise FkError(st, "fk_gelu_tanh")
    return out


def _dtype_code(dt) -> int:
    import torch
    if dt == torch.float32:
        return FK_F32
    if dt == torch.bfloat16:
        return FK_BF16
    raise TypeError("fk operators take float32 or bfloat16")


_GELU_KINDS = {"tanh": FK_GELU_TANH, "none": FK_GELU_ERF}


def gelu(x, out=None, approximate: str = "tanh"):
    """GELU of a contiguous fp32/bf16 CUDA tensor; ``approximate`` is "tanh"
    (the tanh form) or "none" (the exact x * Phi(x)), as in torch's gelu.
    ``out`` may be ``x``."""
    import torch
    _check_tensor(x, "x")
    code = _dtype_code(x.dtype)
    if approximate not in _GELU_KINDS:
        raise ValueError("approximate must be 'tanh' or 'none'")
    if out is None:
        out = torch.empty_like(x)
    _check_tensor(out, "out")
    if out.dtype != x.dtype or out.numel() != x.numel() or out.device != x.device:
        raise ValueError("out must match x in dtype, size and device")
    st = fk_gelu(x.data_ptr(), out.data_ptr(), x.numel(), code, _GELU_KINDS[approximate], _stream_handle(x))
    if st != FK_OK:
        raise FkError(st, "fk_gelu")
    return out


def softmax_rows(x, out=None, plan: SoftmaxPlan | None = None, workspace=None):
    """Softmax over the last dimension of a contiguous fp32/bf16 CUDA tensor.
    `workspace` (a CUDA tensor of at least fk_softmax_rows_workspace bytes)
    makes the call allocation-free; without it the split path allocates its
    workspace stream-ordered."""
    import torch
    _check_tensor(x, "x")
    code = _dtype_code(x.dtype)
    if out is None:
        out = torch.empty_like(x)
    _check_tensor(out, "out")
    if out.dtype != x.dtype or out.shape != x.shape or out.device != x.device:
        raise ValueError("out must match x in dtype, shape and device")
    cols = x.shape[-1] if x.dim() > 0 else 1
    rows = x.numel() // cols if cols else 0
    if workspace is not None:
        _check_tensor(workspace, "workspace")
        st = fk_softmax_rows_ws(x.data_ptr(), out.data_ptr(), rows, cols, code, plan, workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream_handle(x))
    else:
        st = fk_softmax_rows_ex(x.data_ptr(), out.data_ptr(), rows, cols, code, plan, _stream_handle(x))
    if st != FK_OK:
        raise FkError(st, "fk_softmax_rows")
    return out


def softmax_causal(x, scale: float, period: int | None = None, offset: int = 0, out=None,
                   plan: SoftmaxPlan | None = None, skip_masked: bool = False):
    """Scaled, causally masked softmax over the last dimension of a
    contiguous fp32/bf16 CUDA tensor of attention scores [..., T_q, T_k]: row
    i of each [T_q, T_k] block keeps keys j <= i + offset.  `period` defaults
    to T_q (x.shape[-2]); 0 means no mask.  skip_masked: masked outputs are
    not stored (left as they were, or 0)."""
    import torch
    _check_tensor(x, "x")
    code = _dtype_code(x.dtype)
    if x.dim() < 2 and period is None:
        raise ValueError("period is needed for a 1-D tensor")
    if out is None:
        out = torch.empty_like(x)
    _check_tensor(out, "out")
    if out.dtype != x.dtype or out.shape != x.shape or out.device != x.device:
        raise ValueError("out must match x in dtype, shape and device")
    cols = x.shape[-1] if x.dim() > 0 else 1
    rows = x.numel() // cols if cols else 0
    p = x.shape[-2] if period is None else period
    st = fk_softmax_rows_causal_ex(x.data_ptr(), out.data_ptr(), rows, cols, code, scale, p, offset, plan,
                                   _stream_handle(x), FK_SOFTMAX_SKIP_MASKED if skip_masked else 0)
    if st != FK_OK:
        raise FkError(st, "fk_softmax_rows_causal")
    return out


_EPILOGUES = {None: FK_EPILOGUE_NONE, "tanh": FK_EPILOGUE_GELU_TANH, "none": FK_EPILOGUE_GELU_ERF,
              "erf": FK_EPILOGUE_GELU_ERF}


def layernorm(x, eps: float = 1e-5, weight=None, bias=None, gelu: str | None = None, out=None,
              plan: SoftmaxPlan | None = None):
    """LayerNorm over the last dimension of a contiguous fp32/bf16 CUDA
    tensor (as F.layer_norm(x, x.shape[-1:], weight, bias, eps)), then GELU
    when `gelu` is "tanh" or "erf" (or torch's "none", the exact form).
    weight / bias: contiguous fp32 CUDA tensors of x.shape[-1] values."""
    import torch
    _check_tensor(x, "x")
    code = _dtype_code(x.dtype)
    if gelu not in _EPILOGUES:
        raise ValueError("gelu must be None, 'tanh' or 'erf'")
    cols = x.shape[-1] if x.dim() > 0 else 1
    rows = x.numel() // cols if cols else 0
    ptrs = []
    for name, p in (("weight", weight), ("bias", bias)):
        if p is None:
            ptrs.append(0)
            continue
        _check_tensor(p, name)
        if p.dtype != torch.float32 or p.numel() != cols or p.device != x.device:
            raise ValueError(f"{name} must be float32 with x.shape[-1] values on x's device")
        ptrs.append(p.data_ptr())
    if out is None:
        out = torch.empty_like(x)
    _check_tensor(out, "out")
    if out.dtype != x.dtype or out.shape != x.shape or out.device != x.device:
        raise ValueError("out must match x in dtype, shape and device")
    st = fk_layernorm_rows_ex(x.data_ptr(), out.data_ptr(), ptrs[0], ptrs[1], rows, cols, code, eps,
                              _EPILOGUES[gelu], plan, _stream_handle(x))
    if st != FK_OK:
        raise FkError(st, "fk_layernorm_rows")
    return out


def attention(q, k, v, causal: bool = True, scale: float | None = None, out=None):
    """Attention forward on contiguous bf16 CUDA tensors [..., t, d] (all
    leading dimensions are independent slices): softmax(scale q k^T, causal)
    v, with scale = 1/sqrt(d) by default."""
    import math

    import torch
    for name, a in (("q", q), ("k", k), ("v", v)):
        _check_tensor(a, name)
        if a.dtype != torch.bfloat16 or a.shape != q.shape:
            raise ValueError(f"{name} must be bfloat16 with q's shape")
    t, d = q.shape[-2], q.shape[-1]
    bh = q.numel() // (t * d) if t * d else 0
    if out is None:
        out = torch.empty_like(q)
    _check_tensor(out, "out")
    st = fk_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), bh, t, d, int(bool(causal)),
                          1.0 / math.sqrt(d) if scale is None else scale, _stream_handle(q))
    if st != FK_OK:
        raise FkError(st, "fk_attention_fwd")
    return out


__all__ = [
    "FK_OK", "FK_ERR_INVALID_ARG", "FK_ERR_UNSUPPORTED_DTYPE", "FK_ERR_UNSUPPORTED_DEVICE",
    "FK_ERR_CUDA", "FK_F32", "FK_BF16", "FK_GELU_TANH", "FK_GELU_ERF", "FK_PATH_AUTO", "FK_PATH_WARP", "FK_PATH_CTA",
    "FK_PATH_CLUSTER", "FK_PATH_TWOPHASE", "FK_PATH_SPLIT", "FkError", "SoftmaxPlan", "lib", "header_functions",
    "fk_gelu_tanh", "fk_gelu", "fk_copy", "fk_softmax_rows", "fk_softmax_rows_ex", "fk_softmax_rows_plan",
    "fk_softmax_rows_workspace", "fk_softmax_rows_ws", "fk_softmax_rows_noalloc", "fk_softmax_rows_noalloc_cap",
    "fk_softmax_rows_causal", "fk_softmax_rows_causal_ex", "softmax_causal", "FK_SOFTMAX_SKIP_MASKED",
    "fk_layernorm_rows", "fk_layernorm_rows_ex", "fk_layernorm_rows_plan", "layernorm",
    "fk_attention_fwd", "attention", "FK_EPILOGUE_NONE", "FK_EPILOGUE_GELU_TANH",
    "FK_EPILOGUE_GELU_ERF",
    "fk_status_string", "fk_last_cuda_error", "fk_version", "fk_wait_timeouts",
    "fk_wait_selftest", "make_plan", "gelu_tanh", "gelu",
    "softmax_rows",
]
