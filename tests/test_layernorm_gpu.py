"""fk_layernorm_rows on the GPU against the double-precision oracle.

LayerNorm over rows (lecture 6, "GPU Kernels and Triton", sections 6.1-6.2),
optional affine, optional GELU epilogue.  Tolerances, derived from the fp32
arithmetic of the kernels (sums of at most 2^20 terms, x - m1 and the
correction d each exact to a few roundings relative to the row's spread,
rsqrt within 2 ulp): fp32 outputs within 2^-18 (1 + |y|) max(1, |gamma|)
of the oracle; bf16 outputs within 1 ulp of the correctly rounded value, or
within that fp32 bound where a bf16 ulp is smaller (outputs near 0).
"""
import numpy as np
import pytest

import oracle
from _util import Guarded, bf16_ordinal
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2.0 ** -18


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


def run(fk, torch, x, eps=1e-5, gamma=None, beta=None, gelu=None, plan=None, xoff=0, yoff=0, poff=0,
        inplace=False):
    rows, cols = x.shape
    bf16 = x.dtype == np.uint16
    tdt = torch.bfloat16 if bf16 else torch.float32
    host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if bf16 else torch.from_numpy(x)
    dev = torch.device("cuda:0")
    xin = Guarded(torch, x.size, tdt, dev, offset=xoff, fill=host.reshape(-1))
    out = xin if inplace else Guarded(torch, x.size, tdt, dev, offset=yoff)
    params = []
    for p in (gamma, beta):
        params.append(None if p is None else Guarded(torch, cols, torch.float32, dev, offset=poff,
                                                      fill=torch.from_numpy(np.asarray(p, np.float32))))
    epi = {None: fk.FK_EPILOGUE_NONE, "tanh": fk.FK_EPILOGUE_GELU_TANH, "erf": fk.FK_EPILOGUE_GELU_ERF}[gelu]
    st = fk.fk_layernorm_rows_ex(xin.view.data_ptr(), out.view.data_ptr(),
                                 params[0].view.data_ptr() if params[0] else 0,
                                 params[1].view.data_ptr() if params[1] else 0,
                                 rows, cols, fk.FK_BF16 if bf16 else fk.FK_F32, eps, epi, plan,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact(), "write outside the output"
    for g in params:
        assert g is None or g.canaries_intact()
    y = out.view.cpu()
    if bf16:
        return y.view(torch.int16).numpy().view(np.uint16).reshape(rows, cols)
    return y.numpy().reshape(rows, cols)


def _is_nan_bf16(b):
    return ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)


def check(x, y, eps=1e-5, gamma=None, beta=None, gelu=None):
    """Kernel output y (fp32, or bf16 bits) against the oracle on x."""
    xd = oracle.bf16_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)
    ref = oracle.layernorm_rows(xd, eps, gamma, beta, gelu)
    g = np.ones(x.shape[1]) if gamma is None else np.abs(np.asarray(gamma, np.float64))
    tol = TOL * (1.0 + np.abs(ref)) * np.maximum(1.0, g)[None, :]
    if x.dtype == np.uint16:
        assert np.array_equal(_is_nan_bf16(y), np.isnan(ref)), "NaN pattern differs from the oracle"
        ok = ~np.isnan(ref)
        rb = oracle.round_to_bf16(ref)
        ulps = np.abs(bf16_ordinal(y) - bf16_ordinal(rb))
        err = np.abs(oracle.bf16_to_f64(y) - ref)
        bad = ok & (ulps > 1) & (err > tol)
        assert not bad.any(), f"{bad.sum()} bf16 outputs off by more than 1 ulp and the fp32 bound"
        return int(ulps[ok].max()) if ok.any() else 0
    assert np.array_equal(np.isnan(y), np.isnan(ref)), "NaN pattern differs from the oracle"
    ok = ~np.isnan(ref)
    err = np.abs(y.astype(np.float64) - ref)
    ratio = (err / tol)[ok]
    assert ratio.size == 0 or ratio.max() <= 1.0, f"error {ratio.max():.2f} x the bound"
    return float(ratio.max()) if ratio.size else 0.0


def params(cols, seed=0):
    g = np.random.default_rng(seed)
    return ((1.0 + 0.3 * g.standard_normal(cols)).astype(np.float32),
            (0.3 * g.standard_normal(cols)).astype(np.float32))


SHAPES = [(37, 1), (37, 7), (64, 32), (33, 1000), (33, 1023), (17, 1024), (17, 1025), (9, 2048), (9, 2049),
          (9, 4095), (5, 4096), (5, 8193), (3, 16384), (3, 16385), (2, 32768), (2, 32769), (2, 100003),
          (1, 262147)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", SHAPES)
def test_auto_plan(fk, torch_mod, dtype, rows, cols):
    x = synth.layernorm_input(rows, cols, dtype, seed=rows * 31 + cols)
    g, b = params(cols, cols)
    check(x, run(fk, torch_mod, x), 1e-5)
    check(x, run(fk, torch_mod, x, 1e-5, g, b), 1e-5, g, b)


@pytest.mark.parametrize("gelu", ["tanh", "erf"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [100, 2048, 4096, 50000])
def test_gelu_epilogue(fk, torch_mod, gelu, dtype, cols):
    x = synth.layernorm_input(6, cols, dtype, seed=cols + 3)
    g, b = params(cols, 1)
    check(x, run(fk, torch_mod, x, 1e-5, g, b, gelu), 1e-5, g, b, gelu)
    check(x, run(fk, torch_mod, x, 1e-5, None, None, gelu), 1e-5, None, None, gelu)


def _plans(fk, cols, dtype):
    vec = 4 if dtype == "f32" else 8
    plans = [fk.make_plan(fk.FK_PATH_TWOPHASE)]
    for ept in (16, 32):
        for t in (128, 256, 512, 1024):
            if t * ept >= cols:
                plans.append(fk.make_plan(fk.FK_PATH_CTA, threads=t, vpt=ept // vec))
    if cols <= 32 * 8 * vec:
        for t in (32, 64, 128, 256):  # 1, 2, 4 and 8 rows per block
            plans.append(fk.make_plan(fk.FK_PATH_WARP, threads=t, vpt=8))
    return plans


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [1, 100, 1000, 2048, 4096, 20000])
def test_every_path_on_the_same_input(fk, torch_mod, dtype, cols):
    x = synth.layernorm_input(5, cols, dtype, seed=cols)
    g, b = params(cols, 2)
    for p in _plans(fk, cols, dtype):
        check(x, run(fk, torch_mod, x, 1e-5, g, b, "tanh", plan=p), 1e-5, g, b, "tanh")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [64, 1000, 4096, 40000])
def test_misaligned_and_in_place(fk, torch_mod, dtype, cols):
    x = synth.layernorm_input(3, cols, dtype, seed=7)
    g, b = params(cols, 3)
    check(x, run(fk, torch_mod, x, 1e-5, g, b, xoff=1, yoff=1), 1e-5, g, b)
    check(x, run(fk, torch_mod, x, 1e-5, g, b, xoff=1, yoff=3), 1e-5, g, b)
    check(x, run(fk, torch_mod, x, 1e-5, g, b, poff=1), 1e-5, g, b)     # parameters off 16 bytes
    check(x, run(fk, torch_mod, x, 1e-5, g, b, inplace=True), 1e-5, g, b)


@pytest.mark.parametrize("cols", [5, 1000, 4096, 70000])
def test_special_rows(fk, torch_mod, cols):
    x = synth.layernorm_input(6, cols, "f32", seed=cols)
    x[0, :] = 4.25                      # constant -> beta
    x[1, cols // 2] = np.nan            # NaN row
    x[2, cols - 1] = np.inf             # inf row
    x[3, :] = 1000.0 + 0.01 * x[3, :]   # large mean, small spread
    x[4, :] = -7.0
    x[4, 0] = 8.0                       # one outlier
    g, b = params(cols, 4)
    y = run(fk, torch_mod, x, 1e-5, g, b)
    check(x, y, 1e-5, g, b)
    assert np.all(np.abs(y[0] - b) <= 1e-6)
    assert np.all(np.isnan(y[1])) and np.all(np.isnan(y[2]))


def test_large_mean_relative_to_spread(fk, torch_mod):
    """Rows with |mean| / std up to 1e4: the correction d keeps the error at a
    few roundings of |y|, where a single fp32 mean would be off by
    |mean| * 2^-24 / std."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 4096)) * rng.uniform(0.01, 1, (64, 1))
         + rng.uniform(-100, 100, (64, 1))).astype(np.float32)
    check(x, run(fk, torch_mod, x, 0.0), 0.0)
    check(x, run(fk, torch_mod, x, 0.0, plan=fk.make_plan(fk.FK_PATH_TWOPHASE)), 0.0)


@pytest.mark.parametrize("eps", [0.0, 1e-12, 1e-5, 0.5, 100.0])
def test_eps(fk, torch_mod, eps):
    x = synth.layernorm_input(16, 768, "f32", seed=9)
    check(x, run(fk, torch_mod, x, eps), eps)


def test_full_size_workloads(fk, torch_mod):
    """The LayerNorm bench workloads at full size: sampled rows against the
    oracle (affine, and GELU for the bf16 one)."""
    rng = np.random.default_rng(1)
    for name, gelu in (("ln_f32", None), ("ln_gelu_bf16", "tanh")):
        w = synth.WORKLOADS[name]
        x = synth.make(name)
        g, b = synth.layernorm_params(w.shape[1], w.seed)
        y = run(fk, torch_mod, x, 1e-5, g, b, gelu)
        rows = np.unique(np.concatenate([[0, w.shape[0] - 1], rng.integers(0, w.shape[0], 300)]))
        check(x[rows], y[rows], 1e-5, g, b, gelu)
        del x, y


def test_rejects_bad_arguments(fk, torch_mod):
    torch = torch_mod
    x = torch.zeros(8, 64, device="cuda")
    y = torch.empty_like(x)
    g = torch.ones(64, device="cuda")
    s = 0
    F32 = fk.FK_F32
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), 0, 0, 8, 64, F32, -1e-5, 0, s) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), 0, 0, 8, 64, F32, float("nan"), 0, s) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), 0, 0, 8, 64, F32, 1e-5, 3, s) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), 0, 0, 8, 64, 5, 1e-5, 0, s) == fk.FK_ERR_UNSUPPORTED_DTYPE
    # gamma inside the output
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), y.data_ptr() + 256, 0, 8, 64, F32, 1e-5, 0, s) \
        == fk.FK_ERR_INVALID_ARG
    # gamma in pageable host memory, or misaligned
    h = np.ones(64, np.float32)
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), h.ctypes.data, 0, 8, 64, F32, 1e-5, 0, s) \
        == fk.FK_ERR_INVALID_ARG
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), g.data_ptr() + 2, 0, 8, 64, F32, 1e-5, 0, s) \
        == fk.FK_ERR_INVALID_ARG
    assert fk.fk_layernorm_rows(x.data_ptr(), y.data_ptr(), 0, 0, 0, 64, F32, 1e-5, 0, s) == fk.FK_OK
    bad = fk.make_plan(fk.FK_PATH_CLUSTER)
    assert fk.fk_layernorm_rows_ex(x.data_ptr(), y.data_ptr(), 0, 0, 8, 64, F32, 1e-5, 0, bad, s) \
        == fk.FK_ERR_INVALID_ARG


def test_tensor_wrapper_against_torch(fk, torch_mod):
    """Sanity against torch's own GPU layer_norm (+ gelu) on a 3-D tensor."""
    torch = torch_mod
    x = torch.randn(4, 33, 768, device="cuda") * 2 + 1
    w = torch.randn(768, device="cuda") * 0.2 + 1
    b = torch.randn(768, device="cuda") * 0.2
    y = fk.layernorm(x, 1e-5, w, b, gelu="erf")
    t = torch.nn.functional.gelu(torch.nn.functional.layer_norm(x, (768,), w, b, 1e-5))
    assert torch.max(torch.abs(y - t)).item() <= 1e-5
    xb = x.bfloat16()
    yb = fk.layernorm(xb, 1e-5, w, b)
    bits = xb.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1, 768)
    check(bits, yb.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1, 768), 1e-5,
          w.cpu().numpy(), b.cpu().numpy())
