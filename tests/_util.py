"""Test-side helpers: tolerance checks against the oracle and canary-guarded
device buffers (a stand-in for a memory sanitizer: bytes just before and
after every output must be untouched)."""
from __future__ import annotations

import numpy as np

GELU_TOL = 2e-6          # fp32 GELU, max abs error vs the double oracle
SOFTMAX_F32_TOL = 1e-6   # fp32 softmax, max abs error vs the double oracle
BF16_ULPS = 1            # bf16 softmax, ordinal distance to the correctly rounded value

CANARY_ELEMS = 64        # 16-byte aligned margin on both sides


def bf16_ordinal(bits: np.ndarray) -> np.ndarray:
    """Monotone integer encoding of bf16 patterns (+0 and -0 both map to 0)."""
    b = bits.astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


class Guarded:
    """A device buffer of `n` elements with canary margins on both sides.

    `offset` shifts the start by that many elements (to exercise
    misaligned pointers).  `view` is the payload tensor."""

    def __init__(self, torch, n: int, dtype, device, offset: int = 0, fill=None):
        self.torch = torch
        self.n, self.offset = n, offset
        total = CANARY_ELEMS + offset + n + CANARY_ELEMS
        self.buf = torch.empty(total, dtype=dtype, device=device)
        canary = torch.tensor([-12345.5], dtype=dtype) if dtype != torch.uint8 else torch.tensor([0xA5], dtype=dtype)
        self.buf.fill_(canary.item())
        self.canary_value = canary.item()
        self.view = self.buf[CANARY_ELEMS + offset: CANARY_ELEMS + offset + n]
        if fill is not None:
            self.view.copy_(fill)

    def canaries_intact(self) -> bool:
        head = self.buf[:CANARY_ELEMS + self.offset]
        tail = self.buf[CANARY_ELEMS + self.offset + self.n:]
        return bool((head == self.canary_value).all().item()) and bool((tail == self.canary_value).all().item())


def check_softmax_f32(y: np.ndarray, ref64: np.ndarray, x: np.ndarray):
    """fp32 output vs the double oracle: tolerance on finite rows, exact zeros
    at -inf inputs, NaN exactly where the oracle gives NaN."""
    nan_ref = np.isnan(ref64)
    assert np.array_equal(np.isnan(y), nan_ref), "NaN pattern differs from the oracle"
    ok = ~nan_ref
    err = np.abs(y.astype(np.float64)[ok] - ref64[ok])
    assert err.size == 0 or err.max() <= SOFTMAX_F32_TOL, f"max abs err {err.max():.3e}"
    neg = np.isneginf(x) & ok
    assert np.all(y[neg] == 0.0), "-inf input did not give exactly 0"
    return float(err.max()) if err.size else 0.0


def check_softmax_bf16(y_bits: np.ndarray, ref_bits: np.ndarray, x_bits: np.ndarray):
    ref_nan = ((ref_bits & 0x7F80) == 0x7F80) & ((ref_bits & 0x7F) != 0)
    y_nan = ((y_bits & 0x7F80) == 0x7F80) & ((y_bits & 0x7F) != 0)
    assert np.array_equal(y_nan, ref_nan), "NaN pattern differs from the oracle"
    ok = ~ref_nan
    d = np.abs(bf16_ordinal(y_bits[ok]) - bf16_ordinal(ref_bits[ok]))
    assert d.size == 0 or d.max() <= BF16_ULPS, f"max bf16 ulp distance {d.max()}"
    neg = (x_bits == 0xFF80) & ok
    assert np.all(y_bits[neg] == 0x0000), "-inf input did not give exactly +0"
    return int(d.max()) if d.size else 0


def forced_plans(fk, cols, dtype):
    """Every compiled softmax plan that can hold `cols` columns of `dtype`
    ("f32" or "bf16"): CTA and cluster shapes, two-phase with 1..16 blocks,
    split, and the warp path (1 to 8 rows per block) where a row fits a warp."""
    plans = []
    vec = 4 if dtype == "f32" else 8
    for ept in (16, 32):
        for t in (128, 256, 512, 1024):
            if t * ept >= cols:
                plans.append(fk.make_plan(fk.FK_PATH_CTA, threads=t, vpt=ept // vec))
    for ept in (16, 32, 64):
        for t, k in ((128, 2), (128, 3), (256, 5), (128, 8), (128, 16), (512, 16), (1024, 16)):
            if ept == 64 and t > 512:
                continue
            if -(-(-(-cols // vec)) // k) * vec <= t * ept:
                plans.append(fk.make_plan(fk.FK_PATH_CLUSTER, threads=t, cluster=k, vpt=ept // vec))
    for k in (1, 2, 3, 16):
        plans.append(fk.make_plan(fk.FK_PATH_TWOPHASE, cluster=k))
    plans.append(fk.make_plan(fk.FK_PATH_SPLIT))
    if cols <= (1024 if dtype == "f32" else 2048):
        for t in (32, 64, 128, 256):  # 1, 2, 4 and 8 rows per block
            plans.append(fk.make_plan(fk.FK_PATH_WARP, threads=t, vpt=8))
    return plans
