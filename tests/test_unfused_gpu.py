"""The unfused comparison sequences in bench.py compute the same functions
(checked against the oracle), and the fused kernels beat them."""
import numpy as np
import pytest

import bench
import oracle
from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


def test_unfused_sequences_match_the_oracle(cuda_device):
    import torch
    x = synth.normal((1 << 20,), 5.0, seed=31)
    y = bench.gelu_unfused(torch.from_numpy(x).cuda()).cpu().numpy()
    assert np.max(np.abs(y - oracle.gelu_tanh_f64(x.astype(np.float64)))) <= 2e-6
    xs = synth.softmax_input(64, 4096, "f32", neg_inf_frac=0.1, seed=32)
    ys = bench.softmax_unfused(torch.from_numpy(xs).cuda()).cpu().numpy()
    assert np.max(np.abs(ys - oracle.softmax_rows_f64(xs.astype(np.float64)))) <= 1e-6


def test_unfused_leg_runs_and_fused_is_faster(cuda_device):
    import json
    import subprocess
    import sys
    p = subprocess.run([sys.executable, bench.__file__, "--impl", "unfused", "--workload", "cfg3_softmax",
                        "--steps", "5", "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr
    d = json.loads(p.stdout.strip().splitlines()[-1])
    assert d["impl"] == "unfused" and d["speedup_fused_over_unfused"] > 1.5
