"""fk_attention_fwd (tcgen05 tensor cores) against the double-precision
oracle of softmax(scale Q K^T, causal) V.

Tolerance, derived from the kernel's arithmetic: S and O accumulate in fp32
(errors ~1e-6 relative), P is rounded to bf16 before the second product
(relative error <= 2^-9 per weight, so O moves by at most 2^-9 max|v|), and
O is rounded to bf16 (2^-9 |O|).  The test allows twice that:
|O - O_ref| <= 2^-8 (|O_ref| + max |v| of the slice).
"""
import math

import numpy as np
import pytest

import oracle
from _util import Guarded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_mod(cuda_device):
    import torch
    return torch


def _bf16(torch, bits, dev):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)


def run(fk, torch, q, k, v, causal, scale, ooff=0):
    """q, k, v: uint16 bf16 bits [bh, t, d].  Returns O bits.  `ooff` shifts
    the output by that many bf16 elements (8: 16-byte but not 32-byte
    aligned)."""
    bh, t, d = q.shape
    dev = torch.device("cuda:0")
    tq, tk, tv = (_bf16(torch, a, dev) for a in (q, k, v))
    out = Guarded(torch, q.size, torch.bfloat16, dev, offset=ooff)
    st = fk.fk_attention_fwd(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.view.data_ptr(), bh, t, d,
                             int(causal), scale, torch.cuda.current_stream().cuda_stream)
    assert st == fk.FK_OK, fk.fk_status_string(st)
    torch.cuda.synchronize()
    assert out.canaries_intact()
    return out.view.cpu().view(torch.int16).numpy().view(np.uint16).reshape(bh, t, d)


def check(o_bits, q, k, v, causal, scale):
    ref = oracle.attention(*(oracle.bf16_to_f64(a) for a in (q, k, v)), scale, causal)
    o = oracle.bf16_to_f64(o_bits)
    vmax = np.abs(oracle.bf16_to_f64(v)).max(axis=(1, 2))[:, None, None]
    tol = 2.0 ** -8 * (np.abs(ref) + vmax)
    err = np.abs(o - ref)
    assert np.all(np.isfinite(o))
    assert np.all(err <= tol), f"max err {err.max():.3e}, worst ratio {(err / tol).max():.2f}"
    return float((err / tol).max())


def inputs(bh, t, d, seed, sigma=1.0):
    g = np.random.default_rng(seed)
    return tuple(oracle.round_to_bf16(g.standard_normal((bh, t, d)) * sigma) for _ in range(3))


@pytest.mark.parametrize("bh,t,d,causal", [(1, 128, 64, False), (1, 128, 64, True), (2, 256, 64, True),
                                            (2, 256, 128, False), (3, 384, 128, True), (2, 512, 64, False),
                                            (1, 1024, 128, True), (4, 256, 128, True), (2, 384, 64, False),
                                            (1, 640, 128, True), (3, 128, 128, True)])
def test_parity(fk, torch_mod, bh, t, d, causal):
    q, k, v = inputs(bh, t, d, seed=bh * 1000 + t + d)
    scale = 1.0 / math.sqrt(d)
    check(run(fk, torch_mod, q, k, v, causal, scale), q, k, v, causal, scale)
    assert fk.fk_wait_timeouts(reset=True) == 0


@pytest.mark.parametrize("bh,t,d", [(40, 1024, 64), (230, 256, 64), (75, 384, 128), (148, 256, 64)])
def test_persistent_grids(fk, torch_mod, bh, t, d):
    """Non-causal grids of several rounds over the persistent blocks (one per
    SM): a last round of 12 units split into key halves (40 x 1024), a last
    round of 82 units too many to split (230 x 256), a single round of 150
    units of which 2 spill into a split second round, odd query-tile counts
    (75 x 384: the last pair of each slice has one tile), and a grid that
    fills its rounds exactly (148 x 256).  Every slice against the oracle."""
    q, k, v = inputs(bh, t, d, seed=bh * 7 + t)
    scale = 1.0 / math.sqrt(d)
    check(run(fk, torch_mod, q, k, v, False, scale), q, k, v, False, scale)
    assert fk.fk_wait_timeouts(reset=True) == 0


@pytest.mark.parametrize("bh,t,d", [(100, 512, 64), (120, 384, 64), (60, 640, 128)])
def test_persistent_causal_grids(fk, torch_mod, bh, t, d):
    """Causal grids of two rounds over the persistent blocks, the longest
    pairs first: the first S products of a block's next unit go out while its
    current unit's second tile still runs (a pair's first tile has one key
    block fewer), and units of a single query tile (odd query-tile counts,
    384 and 640) shift the three Q slots.  Every slice against the oracle."""
    q, k, v = inputs(bh, t, d, seed=bh * 5 + t + d)
    scale = 1.0 / math.sqrt(d)
    check(run(fk, torch_mod, q, k, v, True, scale), q, k, v, True, scale)
    assert fk.fk_wait_timeouts(reset=True) == 0


@pytest.mark.parametrize("bh,t,d,causal", [(2, 384, 128, True), (40, 1024, 64, False), (3, 256, 64, False)])
def test_output_16_byte_aligned(fk, torch_mod, bh, t, d, causal):
    """An output that is 16-byte but not 32-byte aligned (the entry point
    asks for 16), the split halves' merged rows included (40 x 1024
    non-causal has a split last round)."""
    q, k, v = inputs(bh, t, d, seed=bh + t + d + 3)
    scale = 1.0 / math.sqrt(d)
    check(run(fk, torch_mod, q, k, v, causal, scale, ooff=8), q, k, v, causal, scale)
    assert fk.fk_wait_timeouts(reset=True) == 0


@pytest.mark.parametrize("sigma,scale", [(3.0, 0.125), (1.0, 1.0), (0.2, 0.05)])
def test_score_ranges(fk, torch_mod, sigma, scale):
    """Peaked and flat attention: large scores (the running max moves often)
    and small ones (nearly uniform weights)."""
    q, k, v = inputs(2, 384, 64, seed=int(sigma * 100), sigma=sigma)
    check(run(fk, torch_mod, q, k, v, True, scale), q, k, v, True, scale)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("delta", [-4.0, 3.0, 7.9, 12.0])
def test_running_max_ramps(fk, torch_mod, delta, causal):
    """Scores that rise (or fall) along the keys by `delta` log2 units per
    128-key block: the running max grows a little every block (the output
    is rescaled only once it has outgrown the last rescale by more than
    2^8), by more than that every block, or never after the first."""
    bh, t, d = 2, 1024, 64
    scale = 0.125
    g = np.random.default_rng(int(delta * 10) + 100 + 7 * causal)
    q = np.zeros((bh, t, d))
    q[..., 0] = 1.0
    q[..., 1:] = 0.05 * g.standard_normal((bh, t, d - 1))
    k = 0.05 * g.standard_normal((bh, t, d))
    k[..., 0] = delta / (scale * math.log2(math.e)) * (np.arange(t) / 128.0) + 0.3 * g.standard_normal((bh, t))
    v = g.standard_normal((bh, t, d))
    q, k, v = (oracle.round_to_bf16(a) for a in (q, k, v))
    check(run(fk, torch_mod, q, k, v, causal, scale), q, k, v, causal, scale)
    assert fk.fk_wait_timeouts(reset=True) == 0


def test_constant_values_and_first_row(fk, torch_mod):
    """With every value row equal, every output row is that row; causal row
    0 sees key 0 only."""
    bh, t, d = 2, 256, 128
    q, k, v = inputs(bh, t, d, seed=5)
    vc = np.repeat(v[:, :1], t, axis=1)
    o = oracle.bf16_to_f64(run(fk, torch_mod, q, k, vc, True, 0.1))
    assert np.max(np.abs(o - oracle.bf16_to_f64(vc))) <= 2.0 ** -8 * np.abs(oracle.bf16_to_f64(vc)).max()
    o = oracle.bf16_to_f64(run(fk, torch_mod, q, k, v, True, 0.1))
    v0 = oracle.bf16_to_f64(v[:, 0])
    assert np.all(np.abs(o[:, 0] - v0) <= 2.0 ** -8 * np.abs(v0))


def test_rejects_bad_arguments(fk, torch_mod):
    torch = torch_mod
    x = torch.zeros(2, 256, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    p = x.data_ptr()
    E = fk.FK_ERR_INVALID_ARG
    assert fk.fk_attention_fwd(p, p, p, y.data_ptr(), 2, 200, 64, 1, 0.1, 0) == E      # t not a multiple of 128
    assert fk.fk_attention_fwd(p, p, p, y.data_ptr(), 2, 256, 96, 1, 0.1, 0) == E      # d not 64 / 128
    assert fk.fk_attention_fwd(p, p, p, p, 2, 256, 64, 1, 0.1, 0) == E                 # output overlaps an input
    assert fk.fk_attention_fwd(p, p, p, y.data_ptr(), 2, 256, 64, 2, 0.1, 0) == E      # causal not 0/1
    assert fk.fk_attention_fwd(p, p, p, y.data_ptr(), 2, 256, 64, 1, 0.0, 0) == E      # scale
    assert fk.fk_attention_fwd(p + 2, p, p, y.data_ptr(), 1, 128, 64, 1, 0.1, 0) == E  # misaligned
    assert fk.fk_attention_fwd(p, p, p, y.data_ptr(), 4, 256, 64, 1, 0.1, 0) == E      # past the allocation
    assert fk.fk_attention_fwd(p, p, p, y.data_ptr(), 0, 256, 64, 1, 0.1, 0) == fk.FK_OK


def test_tensor_wrapper_against_torch_sdpa(fk, torch_mod):
    """Sanity against torch's own scaled_dot_product_attention on the GPU."""
    torch = torch_mod
    q, k, v = (torch.randn(2, 4, 512, 128, device="cuda", dtype=torch.bfloat16) for _ in range(3))
    o = fk.attention(q, k, v, causal=True)
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float(), is_causal=True)
    assert torch.max(torch.abs(o.float() - ref)).item() <= 2e-2


@pytest.mark.parametrize("name", ["attn_causal_bf16", "attn_bf16"])
def test_bench_workloads_full_size(fk, torch_mod, name):
    """The attention bench workloads at full size (4 x 16 heads of 2048 x 128)
    in the launch bench.py times: sampled slices against the oracle."""
    from memory_bound_fk_b200 import synth
    w = synth.WORKLOADS[name]
    causal = w.op == "attention"
    qkv = synth.make(name)
    _, bh, t, d = qkv.shape
    scale = 1.0 / math.sqrt(d)
    o = run(fk, torch_mod, qkv[0], qkv[1], qkv[2], causal, scale)
    for sl in (0, bh - 1):
        check(o[sl:sl + 1], qkv[0, sl:sl + 1], qkv[1, sl:sl + 1], qkv[2, sl:sl + 1], causal, scale)
