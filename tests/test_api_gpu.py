"""Behaviour of the entry points on a device: empty inputs, CUDA-graph
capture and replay, streams, and the per-call host cost of the checks."""
import time

import numpy as np
import pytest

import oracle
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


def test_empty_inputs_are_noops(fk, cuda_device):
    import torch
    assert fk.gelu_tanh(torch.empty(0, device="cuda")).numel() == 0
    assert fk.softmax_rows(torch.empty(0, 64, device="cuda")).shape == (0, 64)
    assert fk.softmax_rows(torch.empty(5, 0, device="cuda", dtype=torch.bfloat16)).shape == (5, 0)


def test_graph_capture_and_replay(fk, cuda_device):
    """The entry points only enqueue work on the given stream, so they can
    be captured into a CUDA graph and replayed with new data in place."""
    import torch
    x = torch.from_numpy(synth.softmax_input(64, 131072, "f32", seed=11)).cuda()
    g_in = torch.from_numpy(synth.normal((1 << 20,), 4.0, seed=12)).cuda()
    y = torch.empty_like(x)
    g_out = torch.empty_like(g_in)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm up outside the capture (first-call setup)
        fk.softmax_rows(x, out=y)
        fk.gelu_tanh(g_in, out=g_out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fk.softmax_rows(x, out=y)
        fk.gelu_tanh(g_in, out=g_out)
    for seed in (13, 14):
        x.copy_(torch.from_numpy(synth.softmax_input(64, 131072, "f32", seed=seed)))
        g_in.copy_(torch.from_numpy(synth.normal((1 << 20,), 4.0, seed=seed)))
        graph.replay()
        torch.cuda.synchronize()
        xs = x[:4].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(y[:4].cpu().numpy() - oracle.softmax_rows_f64(xs))) <= 1e-6
        gi = g_in.cpu().numpy()
        assert np.max(np.abs(g_out.cpu().numpy() - oracle.gelu_tanh_f64(gi.astype(np.float64)))) <= 2e-6
    del graph


def test_work_is_ordered_on_the_callers_stream(fk, cuda_device):
    import torch
    s = torch.cuda.Stream()
    x = torch.from_numpy(synth.softmax_input(1024, 4096, "f32", seed=21)).cuda()
    with torch.cuda.stream(s):
        y = fk.softmax_rows(x)
        z = fk.softmax_rows(y)  # depends on y through stream order only
    s.synchronize()
    ref = oracle.softmax_rows_f64(oracle.softmax_rows_f64(x[:8].cpu().numpy().astype(np.float64)))
    assert np.max(np.abs(z[:8].cpu().numpy() - ref)) <= 2e-6


def test_host_cost_per_call_is_small(fk, cuda_device):
    """Argument and pointer checks run on the host for every call; report
    their cost (a tiny row, so the device time does not matter)."""
    import torch
    x = torch.zeros(1, 32, device="cuda")
    y = torch.empty_like(x)
    s = torch.cuda.current_stream().cuda_stream
    for _ in range(100):
        fk.fk_softmax_rows(x.data_ptr(), y.data_ptr(), 1, 32, fk.FK_F32, s)
    torch.cuda.synchronize()
    n = 2000
    t = time.perf_counter()
    for _ in range(n):
        fk.fk_softmax_rows(x.data_ptr(), y.data_ptr(), 1, 32, fk.FK_F32, s)
    dt = (time.perf_counter() - t) / n
    torch.cuda.synchronize()
    print(f"host time per fk_softmax_rows call (incl. ctypes): {dt * 1e6:.2f} us")
    assert dt < 50e-6


def test_fk_copy_reference(fk, cuda_device):
    import torch
    x = torch.randint(0, 1 << 30, ((1 << 22) + 4,), dtype=torch.int32, device="cuda")
    y = torch.zeros_like(x)
    nb = x.numel() * 4
    assert fk.fk_copy(x.data_ptr(), y.data_ptr(), nb, 0) == fk.FK_OK
    torch.cuda.synchronize()
    assert torch.equal(x, y)
    # both data paths (through shared memory while source and destination fit
    # in L2, through registers beyond), ragged last chunk, exact bytes only
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    for nbytes in (l2 // 2 - 48, l2 // 2 + 4096 + 16, 16, 16400):
        a = torch.randint(0, 1 << 30, (nbytes // 4 + 64,), dtype=torch.int32, device="cuda")
        b = torch.full_like(a, -1)
        assert fk.fk_copy(a.data_ptr(), b.data_ptr(), nbytes, 0) == fk.FK_OK
        torch.cuda.synchronize()
        k = nbytes // 4
        assert torch.equal(a[:k], b[:k]) and bool((b[k:] == -1).all()), nbytes
    assert fk.fk_copy(x.data_ptr(), y.data_ptr(), 0, 0) == fk.FK_OK
    assert fk.fk_copy(x.data_ptr(), y.data_ptr(), 24, 0) == fk.FK_ERR_INVALID_ARG      # not a multiple of 16
    assert fk.fk_copy(x.data_ptr() + 4, y.data_ptr(), 32, 0) == fk.FK_ERR_INVALID_ARG  # misaligned
    assert fk.fk_copy(x.data_ptr(), x.data_ptr() + 16, 64, 0) == fk.FK_ERR_INVALID_ARG  # overlap
    assert fk.fk_copy(x.data_ptr(), y.data_ptr(), nb + (1 << 30), 0) == fk.FK_ERR_INVALID_ARG  # past the allocation
