"""Every workload at its full size, through the same entry points and
automatic plans that bench.py times.

Outputs are checked against the oracle on sampled rows (or on every
element, where the oracle finishes in seconds) and, on every row, through
properties that hold at any size: rows sum to one, -inf inputs give exact
zeros, outputs lie in [0, 1], the arg-max is kept.
"""
import numpy as np
import pytest

import oracle
from _util import GELU_TOL, check_softmax_bf16, check_softmax_f32
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


def _to_dev(torch, a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _bits(torch, t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _properties(torch, x, y, sum_tol):
    """Row-level properties on the device, for every row."""
    yf = y.float()
    s = yf.double().sum(dim=1)
    assert float((s - 1.0).abs().max()) <= sum_tol
    assert bool((yf >= 0).all()) and bool((yf <= 1).all())
    neg = torch.isneginf(x.float())
    assert bool((yf[neg] == 0).all())
    # the position of the row maximum keeps the largest output
    am = x.float().argmax(dim=1)
    ymax = yf.max(dim=1).values
    assert bool((yf.gather(1, am[:, None])[:, 0] == ymax).all())


def test_cfg1_softmax_every_row(fk, torch_mod):
    x = synth.make("cfg1_softmax")
    y = fk.softmax_rows(_to_dev(torch_mod, x)).cpu().numpy()
    check_softmax_f32(y, oracle.softmax_rows_f64(x.astype(np.float64)), x)


@pytest.mark.parametrize("name", ["cfg1_gelu", "cfg2_gelu"])
def test_gelu_every_element(fk, torch_mod, name):
    x = synth.make(name)
    y = fk.gelu_tanh(_to_dev(torch_mod, x)).cpu().numpy()
    err = np.abs(y.astype(np.float64) - oracle.gelu_tanh_f64(x.astype(np.float64)))
    assert err.max() <= GELU_TOL


def test_cfg3_softmax(fk, torch_mod):
    torch = torch_mod
    x = synth.make("cfg3_softmax")
    xd = _to_dev(torch, x)
    yd = fk.softmax_rows(xd)
    _properties(torch, xd, yd, 1e-5)
    y = yd.cpu().numpy()
    rows = np.random.default_rng(3).choice(8192, 512, replace=False)
    rows = np.concatenate([[0, 8191], rows])
    check_softmax_f32(y[rows], oracle.softmax_rows_f64(x[rows].astype(np.float64)), x[rows])


def test_cfg4_softmax(fk, torch_mod):
    torch = torch_mod
    x = synth.make("cfg4_softmax")
    xd = _to_dev(torch, x)
    yd = fk.softmax_rows(xd)
    _properties(torch, xd, yd, 2.0 ** -7)
    # first query of every head sees one key: exactly [1, 0, ..., 0]
    first = yd[::2048].float()
    assert bool((first[:, 0] == 1).all()) and bool((first[:, 1:] == 0).all())
    y = _bits(torch, yd)
    del yd, xd
    g = np.random.default_rng(4)
    rows = np.concatenate([np.arange(0, 2048, 97), g.choice(x.shape[0], 2048, replace=False),
                           [x.shape[0] - 1]])
    check_softmax_bf16(y[rows], oracle.softmax_rows_bf16(x[rows]), x[rows])


def test_cfg5_softmax(fk, torch_mod):
    torch = torch_mod
    x = synth.make("cfg5_softmax")
    xd = _to_dev(torch, x)
    yd = fk.softmax_rows(xd)
    _properties(torch, xd, yd, 1e-5)
    y = yd.cpu().numpy()
    rows = np.concatenate([[0, 511], np.random.default_rng(5).choice(512, 30, replace=False)])
    check_softmax_f32(y[rows], oracle.softmax_rows_f64(x[rows].astype(np.float64)), x[rows])


def test_full_configs_in_place(fk, torch_mod):
    torch = torch_mod
    x = synth.make("cfg3_softmax")
    xd = _to_dev(torch, x)
    ref = fk.softmax_rows(xd).clone()
    fk.softmax_rows(xd, out=xd)
    assert torch.equal(xd, ref)
    g = synth.make("cfg2_gelu")
    gd = _to_dev(torch, g)
    gref = fk.gelu_tanh(gd).clone()
    fk.gelu_tanh(gd, out=gd)
    assert torch.equal(gd, gref)
