"""Host-side logic of bench.py, without a GPU: the traffic model against the
lecture's worked example, the whole-job aggregation, the max over ranks
with world-size-2 gloo process groups, and the reference (oracle) arm."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_traffic_model_reproduces_the_lecture_example():
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "fusion_traffic.json")))
    mb = 1 << 20
    t = g["tensor_mb"] * mb
    assert bench.hbm_traffic_bytes(t, g["elementwise_ops"], fused=False) == g["unfused_traffic_mb"] * mb
    assert bench.hbm_traffic_bytes(t, g["elementwise_ops"], fused=True) == g["fused_traffic_mb"] * mb
    assert bench.hbm_traffic_bytes(t, 3, False) // bench.hbm_traffic_bytes(t, 3, True) == g["traffic_ratio"]


def test_workload_bytes_are_one_read_plus_one_write():
    from memory_bound_fk_b200 import synth
    w = synth.WORKLOADS["cfg2_gelu"]
    assert w.algorithmic_bytes == bench.hbm_traffic_bytes(32 << 20, 1, True)
    assert sum(synth.WORKLOADS[n].algorithmic_bytes for n in bench.SUITE) == 9462349824


def test_aggregate_value_counts_every_rank_over_the_slowest():
    # 1 GB per step per rank, 10 steps, 4 ranks, slowest rank 5 ms -> 8000 GB/s
    assert bench.aggregate_value(10 ** 9, 10, 4, 5.0) == pytest.approx(8000.0)
    assert bench.aggregate_value(10 ** 9, 10, 1, 5.0) == pytest.approx(2000.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


_WORKER = r"""
import os, sys, json, datetime
sys.path.insert(0, sys.argv[1])
import torch.distributed as dist
import bench
rank = int(os.environ["RANK"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
local = [10.0 + rank, 3.0 * (1 - rank), 7.5]
out = bench.max_over_ranks(local, int(os.environ["WORLD_SIZE"]))
v = bench.aggregate_value(1000, 2, int(os.environ["WORLD_SIZE"]), out[0])
print(json.dumps({"rank": rank, "max": out, "value": v}))
dist.destroy_process_group()
"""


def test_max_over_ranks_with_two_gloo_ranks(tmp_path):
    port = _free_port()
    script = tmp_path / "worker.py"
    script.write_text(_WORKER)
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=120)
        assert p.returncode == 0, e
        outs.append(json.loads(o.strip().splitlines()[-1]))
    for o in outs:
        assert o["max"] == [11.0, 3.0, 7.5]
        assert o["value"] == pytest.approx(1000 * 2 * 2 / 11e-3 / 1e9)


def _run_bench(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                       capture_output=True, text=True, timeout=300)
    return p


def test_reference_arm_prints_one_json_line():
    p = _run_bench(["--impl", "reference", "--workload", "cfg1_softmax", "--steps", "3",
                    "--warmup", "1", "--reference-budget", "2"])
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_on_a_non_zero_rank_exits_without_work():
    p = _run_bench(["--impl", "reference", "--workload", "cfg1_softmax", "--steps", "2"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_warmup_rule():
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "1"])
    a = bench.parse_args([])
    assert a.warmup >= 3 and a.gpus == 1 and a.impl == "ours"


def test_clock_sampler_parses_nvidia_smi_csv(tmp_path):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    f = open(tmp_path / "c.csv", "w+")
    f.write("1965, 1965, Not Active, Not Active, Not Active, Active\n"
            "1900, 1965, Not Active, Not Active, Not Active, Not Active\n"
            "1800, 1965, Not Active, Not Active, Not Active, Active\n")
    f.flush()
    s.out, s.proc = f, type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout: 0})()
    r = s.stop()
    assert r == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_traffic_model_of_the_unfused_sequences():
    t = 32 << 20
    assert bench.unfused_traffic_bytes("gelu", t) == 18 * t
    assert bench.unfused_traffic_bytes("softmax", t) == 8 * t


def test_source_digest_ignores_comments_and_layout_but_not_code():
    """The digest that ties a profile's DRAM traffic to the kernel sources
    hashes the code only: comments and whitespace may change, code and the
    contents of string literals (inline PTX) may not."""
    src = 'int a = 1; // note\n/* block\n comment */ asm("add.f32 %0, %1; // inside");\n'
    code = bench.code_text(src)
    assert code == 'int a = 1; asm("add.f32 %0, %1; // inside");'
    assert bench.code_text('int  a =\n 1;  /* x */') == bench.code_text('int a = 1; // y')
    assert bench.code_text('int a = 1;') != bench.code_text('int a = 2;')
    assert bench.code_text('asm("mov.u32 %0, 1;")') != bench.code_text('asm("mov.u32 %0, 2;")')


def test_max_error_reports_abs_error_ulps_and_nan_placement():
    import numpy as np
    # fp32: absolute error, NaN compared by position only
    g = np.array([1.0, 2.0, np.nan, 0.0], dtype=np.float32)
    r = np.array([1.0, 2.25, np.nan, 0.0], dtype=np.float32)
    assert bench.max_error(g, r, "f32", chunk=3) == {"max_abs": 0.25, "nan_mismatch": 0}
    r2 = r.copy()
    r2[3] = np.nan
    assert bench.max_error(g, r2, "f32")["nan_mismatch"] == 1
    # bf16: distance in the monotone encoding; -0 and +0 coincide, the
    # smallest subnormals of either sign are 2 apart
    gb = np.array([0x3F80, 0x8000, 0x8001, 0x7FC0], dtype=np.uint16)
    rb = np.array([0x3F81, 0x0000, 0x0001, 0x7FC0], dtype=np.uint16)
    assert bench.max_error(gb, rb, "bf16", chunk=2) == {"max_ulp_bf16": 2, "nan_mismatch": 0}
    assert list(bench.bf16_ordinal(np.array([0xFF80, 0x8000, 0x0000, 0x7F80], dtype=np.uint16))) == \
        [-0x7F80, 0, 0, 0x7F80]


def test_rotation_sets_cover_four_times_the_l2():
    l2 = 126 << 20
    assert bench.rotation_sets(9462349824, l2) == 1          # the suite: one step is 9.5 GB
    assert bench.rotation_sets(4 * l2, l2) == 1
    k = bench.rotation_sets(64 << 20, l2)                     # 32 MiB in + 32 MiB out
    assert k * (64 << 20) >= 4 * l2 and (k - 1) * (64 << 20) < 4 * l2
    assert bench.rotation_sets(1, l2) == 64                   # capped
