"""fk_softmax_rows on the GPU against the double-precision oracle.

Tolerances: fp32 max abs error 1e-6; bf16 within 1 ulp (ordinal distance)
of the correctly rounded double result; -inf inputs give exactly 0; NaN
exactly where the oracle gives NaN.  Every kernel shape (warp, CTA,
cluster, two-phase) is exercised at its capacity boundaries, forced onto
the same inputs, with misaligned pointers, in place, and on special rows.
"""
import numpy as np
import pytest

import oracle
from _util import Guarded, check_softmax_bf16, check_softmax_f32, forced_plans
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


def run(fk, torch, x, plan=None, xoff=0, yoff=0, inplace=False):
    """x: fp32 [rows, cols] or uint16 bf16 bits.  Returns the output (same kind)."""
    rows, cols = x.shape
    bf16 = x.dtype == np.uint16
    tdt = torch.bfloat16 if bf16 else torch.float32
    host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if bf16 else torch.from_numpy(x)
    dev = torch.device("cuda:0")
    xin = Guarded(torch, x.size, tdt, dev, offset=xoff, fill=host.reshape(-1))
    out = xin if inplace else Guarded(torch, x.size, tdt, dev, offset=yoff)
    st = fk.fk_softmax_rows_ex(xin.view.data_ptr(), out.view.data_ptr(), rows, cols,
                               fk.FK_BF16 if bf16 else fk.FK_F32, plan,
                               torch.cuda.current_stream().cuda_stream)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact(), "write outside the output"
    if not inplace:
        assert xin.canaries_intact()
    y = out.view.cpu()
    if bf16:
        return y.view(torch.int16).numpy().view(np.uint16).reshape(rows, cols)
    return y.numpy().reshape(rows, cols)


def check(x, y):
    if x.dtype == np.uint16:
        return check_softmax_bf16(y, oracle.softmax_rows_bf16(x), x)
    return check_softmax_f32(y, oracle.softmax_rows_f64(x.astype(np.float64)), x)


F32_SHAPES = [(37, 1), (37, 2), (37, 31), (37, 32), (37, 33), (37, 127), (37, 128), (37, 129),
              (19, 513), (256, 1000), (33, 1023), (33, 1024), (33, 1025), (9, 4095), (9, 4096),
              (9, 4097), (5, 8193), (5, 16385), (3, 32767), (3, 32768), (3, 32769), (2, 65536),
              (2, 100003), (2, 131072), (2, 131073), (1, 262147), (1, 524288), (1, 524289),
              (1, 1000003), (4096, 64)]
BF16_SHAPES = [(37, 1), (37, 7), (37, 8), (37, 9), (37, 256), (37, 257), (300, 2048), (33, 2047),
               (33, 2049), (9, 4096), (5, 32768), (3, 32769), (2, 131072), (1, 524288),
               (1, 524289)]


@pytest.mark.parametrize("rows,cols", F32_SHAPES)
def test_auto_plan_f32(fk, torch_mod, rows, cols):
    x = synth.softmax_input(rows, cols, "f32", sigma=4.0, neg_inf_frac=0.1, seed=rows * 7 + cols)
    check(x, run(fk, torch_mod, x))


@pytest.mark.parametrize("rows,cols", BF16_SHAPES)
def test_auto_plan_bf16(fk, torch_mod, rows, cols):
    x = synth.softmax_input(rows, cols, "bf16", sigma=8.0, neg_inf_frac=0.3, seed=rows * 11 + cols)
    check(x, run(fk, torch_mod, x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [1, 100, 1000, 1024, 4096, 50000])
def test_every_path_on_the_same_input(fk, torch_mod, dtype, cols):
    rows = 6
    x = synth.softmax_input(rows, cols, dtype, sigma=5.0, neg_inf_frac=0.2, seed=cols)
    for p in forced_plans(fk, cols, dtype):
        check(x, run(fk, torch_mod, x, plan=p))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [64, 1000, 4096, 131072])
def test_misaligned_pointers_take_the_scalar_path(fk, torch_mod, dtype, cols):
    x = synth.softmax_input(3, cols, dtype, sigma=4.0, neg_inf_frac=0.1, seed=5)
    check(x, run(fk, torch_mod, x, xoff=1, yoff=1))
    check(x, run(fk, torch_mod, x, xoff=1, yoff=3))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cols", [1000, 4096, 131072, 600000])
def test_in_place(fk, torch_mod, dtype, cols):
    x = synth.softmax_input(2, cols, dtype, sigma=3.0, neg_inf_frac=0.05, seed=9)
    check(x, run(fk, torch_mod, x, inplace=True))


@pytest.mark.parametrize("cols", [5, 1000, 4096, 131072, 600000])
def test_special_rows(fk, torch_mod, cols):
    x = synth.softmax_input(7, cols, "f32", sigma=2.0, seed=cols)
    x[0, :] = -np.inf                       # all -inf -> NaN row
    x[1, cols // 2] = np.nan                # a NaN -> NaN row
    x[2, cols - 1] = np.inf                 # a +inf -> NaN row
    x[3, :] = 2.5                           # constant -> 1/n
    x[4, cols // 3] += 1000.0               # one huge entry -> one-hot
    x[5, :] = -np.inf                       # causal-like: a single finite entry
    x[5, 0] = 0.25
    y = run(fk, torch_mod, x)
    check(x, y)
    assert np.all(np.isnan(y[:3]))
    assert np.all(np.abs(y[3] - 1.0 / cols) <= 1e-6 / cols + 1e-9)
    assert y[4, cols // 3] == 1.0 and np.count_nonzero(y[4]) == 1
    assert y[5, 0] == 1.0 and np.all(y[5, 1:] == 0.0)


@pytest.mark.parametrize("plan_kind", ["auto", "cluster16", "twophase"])
def test_large_magnitudes_split_across_blocks(fk, torch_mod, plan_kind):
    # Two equal maxima far from zero in different slices of a long row: the
    # merged result must be 0.5 / 0.5 to within the fp32 tolerance, which
    # needs every block's exponentials to be taken relative to its own max.
    cols = 131072
    x = np.full((3, cols), -50.0, np.float32)
    x[0, 10], x[0, cols - 10] = 100.0, 100.0
    x[1] = synth.softmax_input(1, cols, "f32", sigma=4.0, seed=1, shift=100.0)[0]
    x[2] = synth.softmax_input(1, cols, "f32", sigma=1.0, seed=2, shift=-300.0)[0]
    plan = {"auto": None,
            "cluster16": fk.make_plan(fk.FK_PATH_CLUSTER, threads=256, cluster=16),
            "twophase": fk.make_plan(fk.FK_PATH_TWOPHASE, cluster=16)}[plan_kind]
    y = run(fk, torch_mod, x, plan=plan)
    check(x, y)
    assert abs(float(y[0, 10]) - 0.5) <= 1e-6 and abs(float(y[0, cols - 10]) - 0.5) <= 1e-6


@pytest.mark.parametrize("cols", [3, 1000, 4096, 50000])
def test_large_row_maxima(fk, torch_mod, cols):
    # Rows whose max m is large: the single-reference form rounds m * log2(e)
    # and that error (|m log2 e| 2^-24 in the exponent) must not overflow the
    # terms; such rows take the unfolded form.  Maxima from just below the
    # switch (1e7) to FLT_MAX, where m * log2(e) itself overflows, must give
    # the softmax, not NaN, on every path.
    fmax = np.finfo(np.float32).max
    x = synth.softmax_input(8, cols, "f32", sigma=1.0, seed=cols)
    x[0, cols // 2] = fmax                   # one-hot
    x[1, 0], x[1, cols - 1] = fmax, fmax     # even split (cols >= 2)
    x[2, :] = -fmax
    x[2, cols // 3] = 2.5e38                 # one-hot
    x[3, cols - 1] = 5e37                    # one-hot
    x[4, cols - 1] = 1e12                    # one-hot
    x[5] = np.float32(1e9) + np.float32(64) * np.arange(cols) % np.float32(256)  # spacing 64 near 1e9
    x[6] = np.float32(1e7) + (np.arange(cols) % 5).astype(np.float32)      # below the switch: folded
    x[7] = np.float32(2e7) + 2 * (np.arange(cols) % 5).astype(np.float32)  # above it: unfolded
    for p in [None] + forced_plans(fk, cols, "f32"):
        y = run(fk, torch_mod, x, plan=p)
        check(x, y)
        assert y[0, cols // 2] == 1.0 and y[2, cols // 3] == 1.0 and y[4, cols - 1] == 1.0
    b = oracle.round_to_bf16(x.astype(np.float64))
    for p in [None] + forced_plans(fk, cols, "bf16"):
        check(b, run(fk, torch_mod, b, plan=p))


def test_api_rejects_overlap_and_out_of_range(fk, torch_mod):
    import ctypes
    torch = torch_mod
    x = torch.zeros(4096, device="cuda")
    assert fk.fk_softmax_rows(x.data_ptr(), x.data_ptr() + 64, 4, 1000, fk.FK_F32, 0) \
        == fk.FK_ERR_INVALID_ARG
    cuda = ctypes.CDLL("libcuda.so.1")
    base, size = ctypes.c_uint64(), ctypes.c_size_t()
    if cuda.cuMemGetAddressRange_v2(ctypes.byref(base), ctypes.byref(size),
                                    ctypes.c_uint64(x.data_ptr())) != 0:
        pytest.skip("address-range query unavailable")
    y = torch.empty(4096, device="cuda")
    assert fk.fk_softmax_rows(x.data_ptr(), y.data_ptr(), 1 << 30, 4096, fk.FK_F32, 0) \
        == fk.FK_ERR_INVALID_ARG


@pytest.mark.parametrize("cols", [3, 1000, 2048, 4096, 131072, 600000])
def test_bf16_outputs_in_the_subnormal_range_round_correctly(fk, torch_mod, cols):
    # One entry at 0, the rest at -88 .. -95: exp() of those lies below
    # 2^-126, so the correctly rounded bf16 outputs are subnormals down to
    # 2^-133 (or 0); each must still be within 1 ulp of the oracle's rounding.
    x = np.zeros((2, cols), np.float32)
    x[:, 1:] = -88.0 - (np.arange(cols - 1) % 8)
    x[1] = np.roll(x[1], cols // 2)
    xb = synth.f32_to_bf16_bits(x)
    yb = run(fk, torch_mod, xb)
    check(xb, yb)
    ref = oracle.softmax_rows_bf16(xb)
    sub = ((ref & 0x7F80) == 0) & ((ref & 0x7F) != 0)
    assert sub.any()  # the case really reaches bf16 subnormals
    # fp32: the same rows stay within the absolute tolerance
    check(x, run(fk, torch_mod, x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 100), (1, 50000), (2, 600000), (5, 1 << 20),
                                       (7, 1234567)])
def test_split_path(fk, torch_mod, dtype, rows, cols):
    x = synth.softmax_input(rows, cols, dtype, sigma=4.0, neg_inf_frac=0.05, seed=rows + cols)
    p = fk.make_plan(fk.FK_PATH_SPLIT)
    assert fk.fk_softmax_rows_plan(rows, cols, 0 if dtype == "f32" else 1, fk.FK_PATH_SPLIT).chunks >= 1
    check(x, run(fk, torch_mod, x, plan=p))


def test_split_path_special_rows_in_place_and_misaligned(fk, torch_mod):
    cols = 300001
    x = synth.softmax_input(5, cols, "f32", sigma=3.0, seed=77)
    x[0, :] = -np.inf
    x[1, 12345] = np.nan
    x[2, :100000] = -np.inf          # whole chunks with no finite value
    x[3, cols - 1] += 1000.0
    p = fk.make_plan(fk.FK_PATH_SPLIT)
    check(x, run(fk, torch_mod, x, plan=p))
    check(x, run(fk, torch_mod, x, plan=p, inplace=True))
    check(x, run(fk, torch_mod, x, plan=p, xoff=1, yoff=1))


def test_few_long_rows_take_the_split_path_with_a_caller_workspace(fk, torch_mod):
    torch = torch_mod
    rows, cols = 3, 2_000_000
    plan = fk.fk_softmax_rows_plan(rows, cols, fk.FK_F32)
    assert plan.as_dict()["path"] == "split"
    need = fk.fk_softmax_rows_workspace(rows, cols, fk.FK_F32)
    x = torch.from_numpy(synth.softmax_input(rows, cols, "f32", sigma=2.0, seed=5)).cuda()
    ws = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    y1 = fk.softmax_rows(x, workspace=ws)          # allocation-free
    y2 = fk.softmax_rows(x)                         # stream-ordered workspace
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    xs = x[:, :].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(y1.cpu().numpy() - oracle.softmax_rows_f64(xs))) <= 1e-6
    small = torch.empty(max(1, need // 4 - 2), dtype=torch.float32, device="cuda")
    with pytest.raises(fk.FkError):
        fk.softmax_rows(x, workspace=small)
