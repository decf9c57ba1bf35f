"""fk_softmax_rows_causal on the GPU against the double-precision oracle.

The scaled, causally masked softmax (lecture 6, "GPU Kernels and Triton",
section 8): row r keeps columns j <= (r mod period) + offset.  Tolerances as
for fk_softmax_rows: fp32 max abs error 1e-6, bf16 within 1 ulp of the
correctly rounded value; masked columns are exactly +0.  Every kernel path
is forced on the same inputs, aligned and misaligned, and masked inputs are
filled with NaN to show that they never enter the result.
"""
import numpy as np
import pytest

import oracle
from _util import Guarded, bf16_ordinal, check_softmax_bf16, check_softmax_f32, forced_plans
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


def run(fk, torch, x, scale, period, offset=0, plan=None, xoff=0, yoff=0, inplace=False, plain=False):
    rows, cols = x.shape
    bf16 = x.dtype == np.uint16
    tdt = torch.bfloat16 if bf16 else torch.float32
    host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if bf16 else torch.from_numpy(x)
    dev = torch.device("cuda:0")
    xin = Guarded(torch, x.size, tdt, dev, offset=xoff, fill=host.reshape(-1))
    out = xin if inplace else Guarded(torch, x.size, tdt, dev, offset=yoff)
    code = fk.FK_BF16 if bf16 else fk.FK_F32
    s = torch.cuda.current_stream().cuda_stream
    if plain:
        st = fk.fk_softmax_rows_ex(xin.view.data_ptr(), out.view.data_ptr(), rows, cols, code, plan, s)
    else:
        st = fk.fk_softmax_rows_causal_ex(xin.view.data_ptr(), out.view.data_ptr(), rows, cols, code, scale,
                                          period, offset, plan, s)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact(), "write outside the output"
    if not inplace:
        assert xin.canaries_intact()
    y = out.view.cpu()
    if bf16:
        return y.view(torch.int16).numpy().view(np.uint16).reshape(rows, cols)
    return y.numpy().reshape(rows, cols)


def kept_mask(rows, cols, period, offset):
    if period == 0:
        return np.ones((rows, cols), bool)
    q = np.arange(rows) % period + offset
    return np.arange(cols)[None, :] <= q[:, None]


def check(x, y, scale, period, offset):
    """Parity with the oracle, and exact +0 at every masked column (except in
    rows whose kept entries are all -inf: those are NaN throughout, as in
    plain softmax)."""
    rows, cols = x.shape
    keep = kept_mask(rows, cols, period, offset)
    if x.dtype == np.uint16:
        ref = oracle.softmax_rows_causal(x, scale, period, offset)
        check_softmax_bf16(y, ref, np.where(keep, x, np.uint16(0)))
        nan_rows = (((ref & 0x7F80) == 0x7F80) & ((ref & 0x7F) != 0)).any(axis=1)
        masked = ~keep & ~nan_rows[:, None]
        assert np.all(y[masked] == 0x0000)
    else:
        ref = oracle.softmax_rows_causal(x.astype(np.float64), scale, period, offset)
        check_softmax_f32(y, ref, np.where(keep, x, np.float32(0)))
        masked = ~keep & ~np.isnan(ref).any(axis=1)[:, None]
        assert np.all(y[masked] == 0.0) and not np.any(np.signbit(y[masked]))


def poison_masked(x, period, offset):
    """The same input with every masked entry replaced by NaN."""
    keep = kept_mask(*x.shape, period, offset)
    z = x.copy()
    z[~keep] = np.uint16(0x7FC0) if x.dtype == np.uint16 else np.float32(np.nan)
    return z


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols,period,offset", [
    (64, 64, 64, 0), (96, 100, 32, 0), (40, 1000, 40, 960), (24, 1024, 24, 3), (20, 4096, 10, 2000),
    (6, 50000, 3, 20000), (9, 7, 9, 0)])
def test_every_path(fk, torch_mod, dtype, rows, cols, period, offset):
    x = synth.softmax_input(rows, cols, dtype, sigma=5.0, neg_inf_frac=0.05, seed=rows + cols)
    scale = 0.125
    xp = poison_masked(x, period, offset)
    for p in [None] + forced_plans(fk, cols, dtype):
        y = run(fk, torch_mod, xp, scale, period, offset, plan=p)
        check(x, y, scale, period, offset)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [33, 1000, 4097, 131073])
def test_misaligned_and_in_place(fk, torch_mod, dtype, cols):
    rows, period, offset = 5, 5, cols // 2
    x = synth.softmax_input(rows, cols, dtype, sigma=4.0, seed=cols)
    xp = poison_masked(x, period, offset)
    check(x, run(fk, torch_mod, xp, 0.7, period, offset, xoff=1, yoff=1), 0.7, period, offset)
    check(x, run(fk, torch_mod, xp, 0.7, period, offset, xoff=1, yoff=2), 0.7, period, offset)
    check(x, run(fk, torch_mod, xp, 0.7, period, offset, inplace=True), 0.7, period, offset)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [100, 2048, 8192, 200000, 600000])
def test_unmasked_unit_scale_equals_plain_softmax_bitwise(fk, torch_mod, dtype, cols):
    x = synth.softmax_input(3, cols, dtype, sigma=4.0, neg_inf_frac=0.1, seed=cols + 1)
    a = run(fk, torch_mod, x, 1.0, 0)
    b = run(fk, torch_mod, x, 1.0, 0, plain=True)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("scale", [1e-3, 0.0883883, 1.0, 3.0, 40.0])
def test_scales(fk, torch_mod, scale):
    x = synth.softmax_input(128, 128, "f32", sigma=3.0, seed=5)
    check(x, run(fk, torch_mod, x, scale, 128), scale, 128, 0)
    b = synth.softmax_input(128, 128, "bf16", sigma=3.0, seed=6)
    check(b, run(fk, torch_mod, b, scale, 128), scale, 128, 0)


def test_attention_scores_full_size(fk, torch_mod):
    """The attention-score workload (32 x 16 heads of [2048, 2048] bf16
    scores) with the mask generated in the kernel and a scale of 1/8 applied:
    sampled rows, including every head's first and last rows, against the
    oracle.  With scale 1 the result equals plain softmax over the same
    tensor (whose masked entries hold -inf) bit for bit."""
    heads, t = synth.CFG4_HEADS, synth.CFG4_T
    x = synth.make("cfg4_softmax")                 # masked entries hold -inf here
    scale = 0.125
    y = run(fk, torch_mod, x, scale, t)
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([np.arange(heads) * t, np.arange(1, heads + 1) * t - 1,
                                     rng.integers(0, heads * t, 400)]))
    ref = oracle.softmax_rows_causal(x[rows], scale, 0)  # the -inf entries are the mask itself
    check_softmax_bf16(y[rows], ref, x[rows])
    keep = kept_mask(heads * t, t, t, 0)[rows]
    assert np.all(y[rows][~keep] == 0)
    del y
    a = run(fk, torch_mod, x, 1.0, t)
    b = run(fk, torch_mod, x, 1.0, t, plain=True)
    assert np.array_equal(a, b)


def test_rejects_bad_scale(fk, torch_mod):
    torch = torch_mod
    x = torch.zeros(64, 64, device="cuda")
    p = x.data_ptr()
    for s in (0.0, -1.0, float("nan"), float("inf"), -float("inf")):
        assert fk.fk_softmax_rows_causal(p, p, 64, 64, fk.FK_F32, s, 64, 0, 0) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_softmax_rows_causal(p, p, 0, 64, fk.FK_F32, 1.0, 64, 0, 0) == fk.FK_OK
    assert fk.fk_softmax_rows_causal(p, p, 64, 64, 9, 1.0, 64, 0, 0) == fk.FK_ERR_UNSUPPORTED_DTYPE


def test_huge_period_and_offset(fk, torch_mod):
    """period beyond the rows and offset beyond the columns are bounded on
    the host: the results equal the unbounded definition."""
    x = synth.softmax_input(50, 300, "f32", sigma=2.0, seed=8)
    big = 2 ** 62
    check(x, run(fk, torch_mod, x, 0.5, big, 0), 0.5, 50, 0)   # r mod huge = r
    y = run(fk, torch_mod, x, 0.5, 7, big)                     # every column kept
    check(x, y, 0.5, 0, 0)


def test_tensor_wrapper(fk, torch_mod):
    torch = torch_mod
    s = torch.randn(2, 3, 256, 256, device="cuda", dtype=torch.bfloat16)
    y = fk.softmax_causal(s, 0.125)
    bits = s.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1, 256)
    check(bits, y.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1, 256), 0.125, 256, 0)


@pytest.mark.parametrize("period", [1, 2, 3, 5, 7, 100, 1000, 65537, 199999, 200000])
def test_period_division(fk, torch_mod, period):
    """Many short rows: r mod period is taken by multiply-shift division;
    every row's kept count is checked through the oracle."""
    rows, cols, offset = 200000, 16, 3
    x = synth.softmax_input(rows, cols, "f32", sigma=1.0, seed=period)
    check(x, run(fk, torch_mod, x, 0.5, period, offset), 0.5, period, offset)


def test_row_indices_beyond_32_bits(fk, torch_mod):
    """2^32 + 2^20 rows of 2 bf16 zeros, in place (17 GB), period 3: row r
    keeps one column when r mod 3 == 0 (output [1, 0]) and both otherwise
    ([0.5, 0.5]).  Row indices past 2^32 take the 64-bit remainder."""
    torch = torch_mod
    rows, cols = (1 << 32) + (1 << 20), 2
    x = torch.zeros(rows, cols, dtype=torch.bfloat16, device="cuda")
    st = fk.fk_softmax_rows_causal(x.data_ptr(), x.data_ptr(), rows, cols, fk.FK_BF16, 1.0, 3, 0,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    rng = np.random.default_rng(0)
    idx = np.unique(np.concatenate([np.arange(100), (1 << 32) + np.arange(-50, 50), rows - 1 - np.arange(100),
                                    rng.integers(0, rows, 2000)]))
    got = x[torch.from_numpy(idx).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    del x
    torch.cuda.empty_cache()
    one, half = 0x3F80, 0x3F00
    expect = np.where((idx % 3 == 0)[:, None], np.array([[one, 0]], np.uint16), np.array([[half, half]], np.uint16))
    assert np.array_equal(got, expect)


def run_skip(fk, torch, x, scale, period, offset, plan=None, sentinel=7.0):
    """FK_SOFTMAX_SKIP_MASKED into an output pre-filled with `sentinel`."""
    rows, cols = x.shape
    bf16 = x.dtype == np.uint16
    tdt = torch.bfloat16 if bf16 else torch.float32
    host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if bf16 else torch.from_numpy(x)
    dev = torch.device("cuda:0")
    xin = Guarded(torch, x.size, tdt, dev, fill=host.reshape(-1))
    out = Guarded(torch, x.size, tdt, dev)
    out.view.fill_(sentinel)
    st = fk.fk_softmax_rows_causal_ex(xin.view.data_ptr(), out.view.data_ptr(), rows, cols,
                                      fk.FK_BF16 if bf16 else fk.FK_F32, scale, period, offset, plan,
                                      torch.cuda.current_stream().cuda_stream, fk.FK_SOFTMAX_SKIP_MASKED)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact() and xin.canaries_intact()
    y = out.view.cpu()
    if bf16:
        return y.view(torch.int16).numpy().view(np.uint16).reshape(rows, cols)
    return y.numpy().reshape(rows, cols)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [96, 2048, 50000, 200000, 700000])
def test_skip_masked_stores(fk, torch_mod, dtype, cols):
    """Kept outputs equal the oracle's; a masked output is left as it was,
    or is 0 -- and it is always left as it was when its whole 16-byte vector
    is masked (aligned rows), so the masked region costs no writes."""
    rows, period, offset = 6, 6, cols // 3
    x = synth.softmax_input(rows, cols, dtype, sigma=3.0, seed=cols + 11)
    keep = kept_mask(rows, cols, period, offset)
    vec = 4 if dtype == "f32" else 8
    whole = np.zeros_like(keep)
    q = np.arange(rows) % period + offset
    whole[:] = (np.arange(cols)[None, :] // vec * vec) > q[:, None]   # vector starts after the last kept column
    ref = oracle.softmax_rows_causal(x if dtype == "bf16" else x.astype(np.float64), 0.5, period, offset)
    sent = 7.0
    sent_bits = oracle.round_to_bf16(np.array([sent]))[0]
    for p in [None] + forced_plans(fk, cols, dtype):
        y = run_skip(fk, torch_mod, x, 0.5, period, offset, plan=p, sentinel=sent)
        if dtype == "bf16":
            d = np.abs(bf16_ordinal(y[keep]) - bf16_ordinal(ref[keep]))
            assert d.max() <= 1
            assert np.all((y[~keep] == sent_bits) | (y[~keep] == 0))
            assert np.all(y[whole] == sent_bits)
        else:
            assert np.max(np.abs(y[keep].astype(np.float64) - ref[keep])) <= 1e-6
            assert np.all((y[~keep] == sent) | (y[~keep] == 0.0))
            assert np.all(y[whole] == sent)
    # an unknown flag is rejected
    import torch
    t = torch.zeros(4, 4, device="cuda")
    assert fk.fk_softmax_rows_causal_ex(t.data_ptr(), t.data_ptr(), 4, 4, fk.FK_F32, 1.0, 4, 0, None, 0, 2) \
        == fk.FK_ERR_INVALID_ARG
