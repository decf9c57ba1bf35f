"""fk_gelu (both forms, fp32 and bf16) on the GPU against the double oracle.

Tolerances: fp32 max abs error 2e-6 (the GELU bound, both forms); bf16 within
1 ulp of the correctly rounded oracle value, checked exhaustively over all
65536 bf16 inputs, subnormal outputs included.  Limits: GELU(+inf) = +inf,
GELU(-inf) = -0, NaN in gives NaN out.  Ragged sizes, misaligned pointers,
in-place operation and canary margins as for fk_gelu_tanh.
"""
import numpy as np
import pytest

import oracle
from _util import GELU_TOL, Guarded, bf16_ordinal

pytestmark = pytest.mark.gpu

KINDS = ("tanh", "erf")


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


def _kind(fk, kind):
    return fk.FK_GELU_TANH if kind == "tanh" else fk.FK_GELU_ERF


def _ref_f64(kind, x64):
    return oracle.gelu_tanh_f64(x64) if kind == "tanh" else oracle.gelu_erf_f64(x64)


def _run(fk, torch, x_np, dtype_code, kind, xoff=0, yoff=0, inplace=False):
    """x_np: float32 values (fp32) or uint16 bit patterns (bf16)."""
    dev = torch.device("cuda:0")
    if dtype_code == fk.FK_F32:
        tdt, host = torch.float32, torch.from_numpy(x_np)
    else:
        tdt, host = torch.bfloat16, torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16)
    xin = Guarded(torch, x_np.size, tdt, dev, offset=xoff, fill=host)
    out = xin if inplace else Guarded(torch, x_np.size, tdt, dev, offset=yoff)
    st = fk.fk_gelu(xin.view.data_ptr(), out.view.data_ptr(), x_np.size, dtype_code, _kind(fk, kind),
                    torch.cuda.current_stream().cuda_stream)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact()
    if not inplace:
        assert xin.canaries_intact()
    y = out.view.cpu()
    if dtype_code == fk.FK_F32:
        return y.numpy()
    return y.view(torch.int16).numpy().view(np.uint16)


def _check_f32(y, x, kind):
    ref = _ref_f64(kind, x.astype(np.float64))
    fin = np.isfinite(x)
    e = np.abs(y[fin].astype(np.float64) - ref[fin])
    assert e.size == 0 or e.max() <= GELU_TOL, f"max abs err {e.max():.3e}"
    assert np.array_equal(np.isnan(y), np.isnan(x))
    return float(e.max()) if e.size else 0.0


def _is_nan_bf16(b):
    return ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)


def _check_bf16(y_bits, x_bits, kind):
    ref = oracle.round_to_bf16(_ref_f64(kind, oracle.bf16_to_f64(x_bits)))
    assert np.array_equal(_is_nan_bf16(y_bits), _is_nan_bf16(ref)), "NaN pattern differs"
    ok = ~_is_nan_bf16(ref)
    d = np.abs(bf16_ordinal(y_bits[ok]) - bf16_ordinal(ref[ok]))
    assert d.size == 0 or d.max() <= 1, f"max bf16 ulp distance {d.max()}"
    return d


@pytest.mark.parametrize("kind", KINDS)
def test_bf16_exhaustive(fk, torch_mod, kind):
    """Every bf16 bit pattern, so every subnormal, tail and rounding case."""
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    y = _run(fk, torch_mod, x, fk.FK_BF16, kind)
    d = _check_bf16(y, x, kind)
    # nearly all outputs are the correctly rounded value itself
    assert (d == 0).mean() > 0.99
    assert y[0xFF80] == 0x8000              # GELU(-inf) = -0
    assert y[0x7F80] == 0x7F80              # GELU(+inf) = +inf
    assert y[0x0000] == 0x0000 and y[0x8000] == 0x8000


def test_bf16_subnormal_outputs(fk, torch_mod):
    """Negative inputs whose GELU is a bf16 subnormal (below 2^-126): the
    kernel keeps them instead of flushing them to zero."""
    xs = np.arange(-15.0, -9.0, 1.0 / 16).astype(np.float32)
    bits = (xs.view(np.uint32) >> 16).astype(np.uint16)  # exact: 1/16 is the bf16 ulp on [8, 16)
    for kind in KINDS:
        ref = oracle.round_to_bf16(_ref_f64(kind, oracle.bf16_to_f64(bits)))
        sub = ((ref & 0x7F80) == 0) & ((ref & 0x7F) != 0)
        assert sub.sum() >= 4, "precondition: some outputs are subnormal"
        y = _run(fk, torch_mod, bits, fk.FK_BF16, kind)
        _check_bf16(y, bits, kind)
        assert np.all((y[sub] & 0x7F) != 0), f"{kind}: subnormal output flushed"


@pytest.mark.parametrize("kind", KINDS)
def test_f32_dense_grid(fk, torch_mod, kind):
    x = np.linspace(-20.0, 20.0, 4_000_037).astype(np.float32)
    y = _run(fk, torch_mod, x, fk.FK_F32, kind)
    _check_f32(y, x, kind)
    assert np.array_equal(y[x >= 10], x[x >= 10])


@pytest.mark.parametrize("kind", KINDS)
def test_f32_special_values(fk, torch_mod, kind):
    fmax = np.finfo(np.float32).max
    x = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, fmax, -fmax, 1e-45, -1e-45, 1e-38,
                  1e30, -1e30, 1e13, -1e13, 9.0, -9.0, 5.4, -5.4], np.float32)
    y = _run(fk, torch_mod, np.tile(x, 3), fk.FK_F32, kind)[:x.size]
    assert y[0] == 0.0 and not np.signbit(y[0])
    assert y[1] == 0.0
    assert y[2] == np.inf
    assert y[3] == 0.0 and np.signbit(y[3])
    assert np.isnan(y[4])
    assert y[5] == fmax and y[6] == 0.0
    _check_f32(y, x, kind)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("n", [1, 3, 7, 8, 9, 17, 1023, 4097, 262147, (1 << 20) + 5])
def test_ragged_sizes(fk, torch_mod, dtype, kind, n):
    x = (np.random.default_rng(n).standard_normal(n) * 4).astype(np.float32)
    if dtype == "f32":
        _check_f32(_run(fk, torch_mod, x, fk.FK_F32, kind), x, kind)
    else:
        bits = oracle.round_to_bf16(x.astype(np.float64))
        _check_bf16(_run(fk, torch_mod, bits, fk.FK_BF16, kind), bits, kind)


@pytest.mark.parametrize("xoff,yoff", [(1, 1), (3, 3), (5, 5), (7, 7), (1, 2), (0, 3), (6, 0)])
def test_bf16_misaligned_pointers(fk, torch_mod, xoff, yoff):
    x = (np.random.default_rng(11).standard_normal(100_003) * 5).astype(np.float64)
    bits = oracle.round_to_bf16(x)
    for kind in KINDS:
        _check_bf16(_run(fk, torch_mod, bits, fk.FK_BF16, kind, xoff, yoff), bits, kind)


@pytest.mark.parametrize("xoff,yoff", [(1, 1), (2, 2), (1, 2), (0, 3)])
def test_f32_erf_misaligned_pointers(fk, torch_mod, xoff, yoff):
    x = (np.random.default_rng(12).standard_normal(100_003) * 5).astype(np.float32)
    _check_f32(_run(fk, torch_mod, x, fk.FK_F32, "erf", xoff, yoff), x, "erf")


@pytest.mark.parametrize("kind", KINDS)
def test_in_place(fk, torch_mod, kind):
    x = (np.random.default_rng(13).standard_normal(1_000_001) * 6).astype(np.float64)
    bits = oracle.round_to_bf16(x)
    _check_bf16(_run(fk, torch_mod, bits, fk.FK_BF16, kind, inplace=True), bits, kind)
    x32 = x.astype(np.float32)
    _check_f32(_run(fk, torch_mod, x32, fk.FK_F32, kind, inplace=True), x32, kind)


def test_cfg2_size_both_dtypes(fk, torch_mod):
    """The 32 MiB fp32 GELU workload's values, in both forms, and the same
    values as bf16 (half the bytes)."""
    from memory_bound_fk_b200 import synth
    x = synth.make("cfg2_gelu")
    _check_f32(_run(fk, torch_mod, x, fk.FK_F32, "erf"), x, "erf")
    bits = oracle.round_to_bf16(x.astype(np.float64))
    for kind in KINDS:
        _check_bf16(_run(fk, torch_mod, bits, fk.FK_BF16, kind), bits, kind)


def test_tanh_entry_point_is_the_f32_tanh_form(fk, torch_mod):
    torch = torch_mod
    x = torch.randn(1 << 20, device="cuda") * 4
    a, b = torch.empty_like(x), torch.empty_like(x)
    assert fk.fk_gelu_tanh(x.data_ptr(), a.data_ptr(), x.numel(), 0) == fk.FK_OK
    assert fk.fk_gelu(x.data_ptr(), b.data_ptr(), x.numel(), fk.FK_F32, fk.FK_GELU_TANH, 0) == fk.FK_OK
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_tensor_wrapper_and_errors(fk, torch_mod):
    torch = torch_mod
    x = torch.randn(4097, device="cuda", dtype=torch.bfloat16)
    y = fk.gelu(x, approximate="none")
    bits = x.cpu().view(torch.int16).numpy().view(np.uint16)
    _check_bf16(y.cpu().view(torch.int16).numpy().view(np.uint16), bits, "erf")
    with pytest.raises(ValueError):
        fk.gelu(x, approximate="sigmoid")
    with pytest.raises(TypeError):
        fk.gelu(x.half())
    p = x.data_ptr()
    assert fk.fk_gelu(p, p, 16, 7, fk.FK_GELU_TANH, 0) == fk.FK_ERR_UNSUPPORTED_DTYPE
    assert fk.fk_gelu(p, p, 16, fk.FK_BF16, 2, 0) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_gelu(0, 0, 0, fk.FK_BF16, fk.FK_GELU_ERF, 0) == fk.FK_OK  # empty: no-op
    assert fk.fk_gelu(0, p, 16, fk.FK_BF16, fk.FK_GELU_ERF, 0) == fk.FK_ERR_INVALID_ARG


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_both_data_paths_around_the_l2_switch(fk, torch_mod, dtype, kind):
    """Arrays whose input and output together fit in L2 stream through shared
    memory (bulk copies, persistent blocks, a short last chunk); larger ones,
    and inputs under 8 MiB, go through registers.  Both sides of both
    switches, with ragged tails and a misaligned head, against the oracle."""
    l2 = torch_mod.cuda.get_device_properties(0).L2_cache_size
    esize = 4 if dtype == "f32" else 2
    code = fk.FK_F32 if dtype == "f32" else fk.FK_BF16
    limit = l2 // (2 * esize)  # elements at which input + output fill L2
    g = np.random.default_rng(101)
    small = (8 << 20) // esize  # elements at which the input reaches 8 MiB
    for n, off in ((limit - 9, 0), (limit + 13, 0), (limit - 40, 3), (small - 5, 0), (small + 7, 1)):
        x = (g.standard_normal(n) * 5).astype(np.float32)
        if dtype == "f32":
            _check_f32(_run(fk, torch_mod, x, code, kind, xoff=off, yoff=off), x, kind)
        else:
            bits = oracle.round_to_bf16(x.astype(np.float64))
            _check_bf16(_run(fk, torch_mod, bits, code, kind, xoff=off, yoff=off), bits, kind)
