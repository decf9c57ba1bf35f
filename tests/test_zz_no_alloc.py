"""fk_softmax_rows_noalloc: softmax for callers that cannot allocate device
memory (a framework holding nearly all of it, allocation-free hot loops).
Its scratch is a fixed array inside the library; its output must match the
existing entry point's (fk_softmax_rows_ws with caller workspace) on the
split path, which is the path that needs scratch, on two calls in a row.

This file is collected last on purpose.  It also passes when run alone in a
fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(fk, x, y, rows, cols, dtype, stream):
    f = fk.lib().fk_softmax_rows_noalloc        # straight through the C ABI
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_size_t, ctypes.c_int,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f(x, y, rows, cols, dtype, stream)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(fk, cuda_device, dtype):
    import torch
    code = fk.FK_F32 if dtype == "f32" else fk.FK_BF16
    s = torch.cuda.current_stream().cuda_stream
    # two different split-path shapes, one after the other
    for call, (rows, cols, seed) in enumerate([(3, 2_000_000, 41), (2, 5_000_001, 42)]):
        assert fk.fk_softmax_rows_plan(rows, cols, code).as_dict()["path"] == "split"
        host = synth.softmax_input(rows, cols, dtype, sigma=3.0, neg_inf_frac=0.05, seed=seed)
        if dtype == "f32":
            x = torch.from_numpy(host).cuda()
        else:
            x = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16).cuda()
        y_ref = torch.empty_like(x)
        y = torch.full_like(x, float("nan"))
        need = fk.fk_softmax_rows_workspace(rows, cols, code)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        assert fk.fk_softmax_rows_ws(x.data_ptr(), y_ref.data_ptr(), rows, cols, code, None,
                                     ws.data_ptr(), need, s) == fk.FK_OK
        assert _noalloc(fk, x.data_ptr(), y.data_ptr(), rows, cols, code, s) == fk.FK_OK, call
        torch.cuda.synchronize()
        if dtype == "f32":
            d = (y.double() - y_ref.double()).abs().max().item()
            assert d <= 1e-6
            # every row against the oracle (fp32 tolerance 1e-6)
            ref = oracle.softmax_rows_f64(host.astype(np.float64))
            assert np.max(np.abs(y.cpu().numpy().astype(np.float64) - ref)) <= 1e-6
        else:
            a = y.view(torch.int16).cpu().numpy().view(np.uint16)
            b = y_ref.view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.max(np.abs(_ordinal(a) - _ordinal(b))) <= 1
            # every row against the correctly rounded oracle: within 1 bf16
            # ulp, and exactly +0 where the input is -inf
            ref = oracle.softmax_rows_bf16(host)
            assert np.max(np.abs(_ordinal(a) - _ordinal(ref))) <= 1
            neg_inf = host == 0xFF80
            assert neg_inf.any() and np.all(a[neg_inf] == 0)


def _ordinal(bits):
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def test_noalloc_on_the_other_paths_and_arguments(fk, cuda_device):
    import torch
    s = torch.cuda.current_stream().cuda_stream
    x = torch.from_numpy(synth.softmax_input(64, 4096, "f32", seed=43)).cuda()
    y = torch.empty_like(x)
    assert _noalloc(fk, x.data_ptr(), y.data_ptr(), 64, 4096, fk.FK_F32, s) == fk.FK_OK
    torch.cuda.synchronize()
    assert torch.equal(y, fk.softmax_rows(x))
    assert _noalloc(fk, 0, 0, 0, 4096, fk.FK_F32, s) == fk.FK_OK
    assert _noalloc(fk, x.data_ptr(), y.data_ptr(), 64, 4096, 7, s) == fk.FK_ERR_UNSUPPORTED_DTYPE


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_batches_rows_when_the_scratch_is_small(fk, cuda_device, dtype):
    """With 1200 of the array's pairs, 80 split-path rows of 2^22 columns run
    as a batch of 75 rows (16 chunks each) and a last batch of 5 (171 chunks
    each, planned for 5 rows): every row against the oracle, the rows at the
    batch boundary among them.  A capacity that cannot hold a batch is
    refused before anything is written."""
    import torch
    code = fk.FK_F32 if dtype == "f32" else fk.FK_BF16
    rows, cols, cap = 80, 1 << 22, 1200
    assert fk.fk_softmax_rows_plan(rows, cols, code).as_dict()["path"] == "split"
    s = torch.cuda.current_stream().cuda_stream
    host = synth.softmax_input(rows, cols, dtype, sigma=3.0, neg_inf_frac=0.01, seed=44)
    if dtype == "f32":
        x = torch.from_numpy(host).cuda()
    else:
        x = torch.from_numpy(host.view(np.int16)).cuda()
    y = torch.full_like(x, 7)
    assert fk.fk_softmax_rows_noalloc_cap(x.data_ptr(), y.data_ptr(), rows, cols, code, 100, s) == \
        fk.FK_ERR_INVALID_ARG
    assert fk.fk_softmax_rows_noalloc_cap(x.data_ptr(), y.data_ptr(), rows, cols, code, 0, s) == \
        fk.FK_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((y == 7).all()), "a refused call wrote output"
    assert fk.fk_softmax_rows_noalloc_cap(x.data_ptr(), y.data_ptr(), rows, cols, code, cap, s) == fk.FK_OK
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    for r in (0, 1, 37, 74, 75, 76, 79):
        if dtype == "f32":
            ref = oracle.softmax_rows_f32(host[r:r + 1])[0]
            assert np.max(np.abs(got[r].astype(np.float64) - ref)) <= 1e-6, r
        else:
            ref = oracle.softmax_rows_bf16(host[r:r + 1])[0]
            assert np.max(np.abs(_ordinal(got[r].view(np.uint16)) - _ordinal(ref))) <= 1, r
