"""fk_gelu_tanh on the GPU against the double-precision oracle.

Tolerance: max abs error 2e-6 for fp32 (every finite input), exact limits at
+-inf, NaN propagation.  Sizes span many thread blocks and ragged tails;
pointers are offset to exercise the scalar head/tail and the fully scalar
path; in-place operation; canary margins around every output.
"""
import numpy as np
import pytest

import oracle
from _util import GELU_TOL, Guarded

pytestmark = pytest.mark.gpu


def _run(fk, torch, x_np, xoff=0, yoff=0, inplace=False):
    dev = torch.device("cuda:0")
    xin = Guarded(torch, x_np.size, torch.float32, dev, offset=xoff, fill=torch.from_numpy(x_np))
    if inplace:
        out = xin
    else:
        out = Guarded(torch, x_np.size, torch.float32, dev, offset=yoff)
    st = fk.fk_gelu_tanh(xin.view.data_ptr(), out.view.data_ptr(), x_np.size,
                         torch.cuda.current_stream().cuda_stream)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact()
    if not inplace:
        assert xin.canaries_intact()
        assert np.array_equal(xin.view.cpu().numpy().view(np.uint32), x_np.view(np.uint32)), "input modified"
    return out.view.cpu().numpy()


def _err(y, x):
    ref = oracle.gelu_tanh_f64(x.astype(np.float64))
    fin = np.isfinite(x)
    return np.abs(y[fin].astype(np.float64) - ref[fin])


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


@pytest.mark.parametrize("name", ["cfg1_gelu", "cfg2_gelu"])
def test_gelu_configs_full(fk, torch_mod, name):
    from memory_bound_fk_b200 import synth
    x = synth.make(name)
    y = _run(fk, torch_mod, x)
    e = _err(y, x)
    assert e.max() <= GELU_TOL, e.max()


def test_gelu_dense_grid(fk, torch_mod):
    x = np.linspace(-20.0, 20.0, 4_000_037).astype(np.float32)
    y = _run(fk, torch_mod, x)
    e = _err(y, x)
    assert e.max() <= GELU_TOL, e.max()
    # large positive inputs are returned unchanged, large negative give ~0
    assert np.array_equal(y[x >= 10], x[x >= 10])
    assert np.all(np.abs(y[x <= -10]) < 1e-30)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 7, 8, 15, 16, 17, 1023, 1024, 1025, 4097,
                               262147, (1 << 20) + 5, 3 * 2 ** 21 + 1])
def test_gelu_ragged_sizes(fk, torch_mod, n):
    x = (np.random.default_rng(n).standard_normal(n) * 4).astype(np.float32)
    e = _err(_run(fk, torch_mod, x), x)
    assert e.max() <= GELU_TOL


@pytest.mark.parametrize("xoff,yoff", [(1, 1), (2, 2), (3, 3), (1, 2), (0, 3), (2, 0)])
def test_gelu_misaligned_pointers(fk, torch_mod, xoff, yoff):
    x = (np.random.default_rng(7).standard_normal(100_003) * 5).astype(np.float32)
    e = _err(_run(fk, torch_mod, x, xoff, yoff), x)
    assert e.max() <= GELU_TOL


def test_gelu_in_place(fk, torch_mod):
    x = (np.random.default_rng(3).standard_normal(1_000_001) * 6).astype(np.float32)
    e = _err(_run(fk, torch_mod, x, inplace=True), x)
    assert e.max() <= GELU_TOL


def test_gelu_special_values(fk, torch_mod):
    fmax = np.finfo(np.float32).max
    x = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, fmax, -fmax, 1e-45, -1e-45, 1e-38,
                  1e30, -1e30, 1e13, -1e13, 9.0, -9.0, 5.4, -5.4], np.float32)
    y = _run(fk, torch_mod, np.tile(x, 3))[:x.size]
    assert y[0] == 0.0 and y[1] == 0.0
    assert y[2] == np.inf
    assert y[3] == 0.0 and np.signbit(y[3])
    assert np.isnan(y[4])
    assert y[5] == fmax and y[6] == 0.0
    e = _err(y, x)
    assert e.max() <= GELU_TOL


def test_gelu_rejects_out_of_range_size(fk, torch_mod):
    import ctypes
    torch = torch_mod
    x = torch.zeros(1 << 20, device="cuda")
    y = torch.empty_like(x)
    # Only meaningful (and only safe) when the driver's address-range query
    # works on this pointer; then a size past the allocation is an error.
    cuda = ctypes.CDLL("libcuda.so.1")
    base, size = ctypes.c_uint64(), ctypes.c_size_t()
    fn = cuda.cuMemGetAddressRange_v2
    if fn(ctypes.byref(base), ctypes.byref(size), ctypes.c_uint64(x.data_ptr())) != 0:
        pytest.skip("address-range query unavailable")
    st = fk.fk_gelu_tanh(x.data_ptr(), y.data_ptr(), x.numel() + (1 << 40), 0)
    assert st == fk.FK_ERR_INVALID_ARG
    # pageable host memory is not device memory
    h = np.zeros(16, np.float32)
    assert fk.fk_gelu_tanh(h.ctypes.data, y.data_ptr(), 16, 0) == fk.FK_ERR_INVALID_ARG
