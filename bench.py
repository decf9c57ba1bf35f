#!/usr/bin/env python
"""Throughput of the fused memory-bound operators on B200, as achieved HBM GB/s.

One step = one pass of the whole hot path over one batch of synthetic input:
tanh-GELU over 8,388,608 fp32 values (32 MiB), then row softmax over
8192 x 4096 fp32, 1,048,576 x 2048 bf16 (32 x 16 heads of 2048 x 2048 causal
attention scores) and 512 x 131072 fp32 -- every workload of 32 MB and more.
The bytes counted are the algorithmic ones: one read of every input element
plus one write of every output element (the fused-kernel traffic of
"Lecture 6: GPU Kernels and Triton", cs336.sjfarmltd.com, section 1.1).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  Timing: W untimed steps, then K steps
between a barrier + device synchronisation on both sides, CUDA events on
the launching stream, the maximum over ranks.  Every step reads 4.7 GB, far
more than the 126 MB L2, so no step finds its inputs in L2.  For N > 1
(torchrun, one process per GPU) every rank runs the same full workload on
its own GPU (independent replicas, weak scaling, no collective on the data
path) and `value` counts the bytes of all ranks.

`--impl reference` times the double-precision CPU oracle (the test checker,
not a GPU code path) on a bounded sample of the same workload on the host
cores; it is a deliberately slow baseline, not a target.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "achieved HBM GB/s (and % of ~8 TB/s) for row softmax and GELU at 1 B200"
UNIT = "GB/s"
SUITE = ["cfg2_gelu", "cfg3_softmax", "cfg4_softmax", "cfg5_softmax"]
SPEC_HBM_GBS = 8000.0          # nominal B200 HBM3e bandwidth
FALLBACK_HBM_GBS = 6650.0      # earlier copy measurement on this B200 pool


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------- host logic

def kernel_name(w, plan: dict) -> str:
    """The libfk kernel a workload's plan launches."""
    t = "bf16" if w.dtype == "bf16" else "float"
    if w.op in ("gelu", "gelu_erf"):
        return f"gelu_kernel<{t},{'tanh' if w.op == 'gelu' else 'erf'}>"
    if w.op.startswith("layernorm"):
        epi = ",gelu_tanh" if w.op == "layernorm_gelu" else ""
        vec = 8 if w.dtype == "bf16" else 4
        if plan["path"] == "warp":
            return f"layernorm_warp_kernel<{t},vpt={plan['vpt']}{epi}>"
        if plan["path"] == "cta":
            return f"layernorm_block_kernel<{t},{plan['threads']},ept={plan['vpt'] * vec}{epi}>"
        return f"layernorm_stream_kernel<{t}{epi}>"
    sc = ",scaled" if w.op.startswith("softmax_causal") else ""
    vec = 8 if w.dtype == "bf16" else 4
    p = plan["path"]
    if p == "warp":
        return f"softmax_warp_kernel<{t},vpt={plan['vpt']}{sc}>"
    if p == "cta":
        return f"softmax_block_kernel<{t},{plan['threads']},ept={plan['vpt'] * vec}{sc}>"
    if p == "cluster":
        return (f"softmax_cluster_kernel<{t},{plan['threads']},ept={plan['vpt'] * vec}{sc}>"
                f" x cluster {plan['cluster']}")
    if p == "split":
        return f"softmax_split_stats_kernel + softmax_split_norm_kernel<{t}{sc}>"
    return f"softmax_twophase_kernel<{t},cluster={plan['cluster']}{sc}>"


LN_EPS = 1e-5


def launch_workload(fk, w, xp: int, yp: int, shape, stream: int, params=None) -> int:
    """One call of a workload's operator through the C ABI; the status.
    The causal softmax treats every `cols` rows as one block of queries
    against `cols` keys (scale 1: the result equals plain softmax over the
    same scores with the masked entries at -inf).  LayerNorm takes
    `params` = (gamma pointer, beta pointer) and eps 1e-5."""
    code = fk.FK_BF16 if w.dtype == "bf16" else fk.FK_F32
    if w.op.startswith("layernorm"):
        epi = fk.FK_EPILOGUE_GELU_TANH if w.op == "layernorm_gelu" else fk.FK_EPILOGUE_NONE
        return fk.fk_layernorm_rows(xp, yp, params[0], params[1], shape[0], shape[1], code, LN_EPS, epi, stream)
    if w.op in ("gelu", "gelu_erf"):
        kind = fk.FK_GELU_TANH if w.op == "gelu" else fk.FK_GELU_ERF
        return fk.fk_gelu(xp, yp, shape[0], code, kind, stream)
    rows, cols = shape
    if w.op == "softmax_causal":
        return fk.fk_softmax_rows_causal(xp, yp, rows, cols, code, 1.0, cols, 0, stream)
    if w.op == "softmax_causal_skip":
        return fk.fk_softmax_rows_causal_ex(xp, yp, rows, cols, code, 1.0, cols, 0, None, stream,
                                            fk.FK_SOFTMAX_SKIP_MASKED)
    return fk.fk_softmax_rows(xp, yp, rows, cols, code, stream)


def workload_bytes(w, shape) -> int:
    from memory_bound_fk_b200 import synth
    return synth.algorithmic_bytes(w.op, w.itemsize, tuple(shape))


def hbm_traffic_bytes(tensor_bytes: int, n_elementwise_ops: int, fused: bool) -> int:
    """HBM bytes of n elementwise ops over one tensor: each unfused op reads
    and writes the whole tensor; the fused kernel reads it once and writes
    once."""
    return 2 * tensor_bytes if fused else 2 * n_elementwise_ops * tensor_bytes


def rotation_sets(bytes_step: int, l2_bytes: int, max_sets: int = 64) -> int:
    """Buffer sets a step rotates through so that its footprint over the
    sets is at least 4x the L2 size (1 when one step already is)."""
    if bytes_step <= 0 or bytes_step >= 4 * l2_bytes:
        return 1
    return min(max_sets, -(-4 * l2_bytes // bytes_step))


def workload_list(name: str) -> list[str]:
    return SUITE if name == "suite" else [name]


def describe(names: list[str]) -> str:
    from memory_bound_fk_b200 import synth
    return " + ".join(f"{n}: {synth.WORKLOADS[n].recipe}" for n in names)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values: list[float], world: int, device=None) -> list[float]:
    """Element-wise maximum of `values` over all ranks (identity for 1 rank)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def aggregate_value(bytes_per_step_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job GB/s: bytes moved by all ranks / slowest rank's time."""
    return bytes_per_step_per_rank * steps * world / (max_ms * 1e-3) / 1e9


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if d.get("hbm_gbs"):
            return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


# Sources each kernel family is compiled from (its profile stays valid while
# these are unchanged).
_FAMILY_SOURCES = {
    "gelu": ["fk_gelu.cu", "fk_gelu.cuh", "fk_f32x2.cuh", "fk_common.cuh"],
    "softmax": ["fk_softmax.cu", "fk_rows.cuh", "fk_common.cuh", "fk_sync.cuh", "fk_plan.cpp"],
    "layernorm": ["fk_layernorm.cu", "fk_rows.cuh", "fk_common.cuh", "fk_gelu.cuh", "fk_f32x2.cuh", "fk_plan.cpp"],
    "attention": ["fk_attention.cu", "fk_tc.cuh", "fk_sync.cuh", "fk_common.cuh"],
}


def kernel_family(op: str) -> str:
    for fam in ("gelu", "softmax", "layernorm", "attention"):
        if op.startswith(fam):
            return fam
    raise KeyError(op)


def code_text(src: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace collapsed:
    what the compiler sees, so that a comment edit does not count as a kernel
    change.  String literals (inline PTX) are kept, so a `//` inside one is
    not taken for a comment; runs of whitespace are collapsed there too,
    which changes nothing ptxas reads."""
    out, pos = [], 0
    for m in re.finditer(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', src, re.S):
        out.append(src[pos:m.start()])
        out.append(m.group(0) if m.group(0).startswith('"') else " ")
        pos = m.end()
    out.append(src[pos:])
    return " ".join("".join(out).split())


def csrc_digest(family: str | None = None) -> str:
    """Digest of the code (comments and layout excluded) of the kernel
    sources of one family (all of csrc/ if None), with the shared internal
    header and the public header."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "memory_bound_fk_b200", "csrc")
    if family is None:
        files = sorted(glob.glob(os.path.join(csrc, "*")))
    else:
        files = [os.path.join(csrc, f) for f in _FAMILY_SOURCES[family] + ["fk_internal.h"]]
    files.append(os.path.join(ROOT, "include", "fk.h"))
    for p in files:
        with open(p, encoding="utf-8") as f:
            h.update(os.path.basename(p).encode())
            h.update(code_text(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch recorded by an ncu capture in profiles/, if the
    kernel family's sources have not changed since (else None)."""
    from memory_bound_fk_b200 import synth
    digest = csrc_digest(kernel_family(synth.WORKLOADS[workload].op))
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(p).read()
        for m in re.finditer(r"traffic:\s*workload=(\w+)\s+bytes_per_launch=(\d+)\s+csrc=(\w+)", text):
            if m.group(1) == workload and m.group(3) == digest:
                return int(m.group(2)), os.path.relpath(p, ROOT)
    return None, None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id: str, period_ms: int = 20):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", str(period_ms)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def wait_ready(self, timeout_s: float = 3.0) -> None:
        """Block until nvidia-smi has written its first reading (it takes a
        few hundred ms to start), so that a short timed region still has a
        reading next to it."""
        t0 = time.monotonic()
        while self.proc is not None and time.monotonic() - t0 < timeout_s:
            self.out.flush()
            if os.path.getsize(self.out.name) > 0:
                return
            time.sleep(0.02)

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        sm, smax, reasons = [], [], set()
        for line in self.out.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, parts[2:]):
                if val.lower() == "active":
                    reasons.add(name)
        os.unlink(self.out.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- oracle timing

def oracle_sample_plan(names, inputs, budget_s: float, threads: int):
    """Pick the leading fraction f of every workload whose oracle run takes
    about budget_s on `threads` host threads (calibrated on 1/256)."""
    import numpy as np  # noqa: F401
    cal = oracle_run(names, inputs, 1.0 / 256, threads)
    f = min(1.0, max(1.0 / 4096, budget_s / max(cal["seconds"] * 256, 1e-9)))
    return f


def _slice(name, arr, frac):
    if arr.ndim == 1:
        n = max(1, int(arr.shape[0] * frac))
        return arr[:n]
    r = max(1, int(round(arr.shape[0] * frac)))
    return arr[:r]


def oracle_run(names, inputs, frac, threads, keep=False):
    """The oracle over the leading fraction `frac` of every workload, timed;
    with keep=True its outputs (fp32 values or bf16 bit patterns, rounded
    once from double) are returned too, for the max-error check."""
    import oracle
    from memory_bound_fk_b200 import synth
    total_bytes, elems, outputs, per = 0, 0, {}, {}
    t0 = time.perf_counter()
    for n in names:
        w = synth.WORKLOADS[n]
        x = _slice(n, inputs[n], frac)
        tw = time.perf_counter()
        if w.op in ("gelu", "gelu_erf"):
            f64 = oracle.gelu_tanh_f64 if w.op == "gelu" else oracle.gelu_erf_f64
            if w.dtype == "f32":
                y = oracle.round_to_f32(f64(x.astype(np.float64), nthreads=threads))
            else:
                y = oracle.round_to_bf16(f64(oracle.bf16_to_f64(x), nthreads=threads))
        elif w.op.startswith("softmax_causal"):
            y = oracle.softmax_rows_causal(x, 1.0, x.shape[1], 0, nthreads=threads)
        elif w.op.startswith("layernorm"):
            g, b = synth.layernorm_params(x.shape[1], w.seed)
            y = oracle.layernorm_rows(x, LN_EPS, g, b, "tanh" if w.op == "layernorm_gelu" else None,
                                      nthreads=threads)
        elif w.dtype == "f32":
            y = oracle.softmax_rows_f32(x, nthreads=threads)
        else:
            y = oracle.softmax_rows_bf16(x, nthreads=threads)
        per[n] = {"seconds": time.perf_counter() - tw, "elements": int(x.size),
                  "bytes": workload_bytes(w, x.shape)}
        if keep:
            outputs[n] = y
        total_bytes += workload_bytes(w, x.shape)
        elems += x.size
    dt = time.perf_counter() - t0
    return {"seconds": dt, "bytes": total_bytes, "elements": elems, "outputs": outputs, "per_workload": per}


def bf16_ordinal(bits: np.ndarray) -> np.ndarray:
    """Monotone integer encoding of bf16 bit patterns (adjacent values differ by 1)."""
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def max_error(gpu: np.ndarray, ref: np.ndarray, dtype: str, chunk: int = 1 << 24) -> dict:
    """Largest deviation of GPU outputs from the oracle's correctly rounded
    outputs: absolute error for fp32, distance in bf16 ulps for bf16.  NaN
    must sit at the same places on both sides.  Works through the arrays in
    pieces of `chunk` elements to bound host memory."""
    g_all, r_all = gpu.reshape(-1), ref.reshape(-1)
    worst, nan_mismatch = 0, 0
    for i in range(0, g_all.size, chunk):
        if dtype == "bf16":
            g, r = g_all[i:i + chunk].view(np.uint16), r_all[i:i + chunk].view(np.uint16)
            gn, rn = (g & 0x7FFF) > 0x7F80, (r & 0x7FFF) > 0x7F80
            d = np.where(gn | rn, 0, np.abs(bf16_ordinal(g) - bf16_ordinal(r)))
            worst = max(worst, int(d.max(initial=0)))
        else:
            g, r = g_all[i:i + chunk].astype(np.float64), r_all[i:i + chunk].astype(np.float64)
            gn, rn = np.isnan(g), np.isnan(r)
            d = np.where(gn | rn, 0.0, np.abs(g - r))
            worst = max(worst, float(d.max(initial=0.0)))
        nan_mismatch += int(np.count_nonzero(gn != rn))
    key = "max_ulp_bf16" if dtype == "bf16" else "max_abs"
    return {key: worst, "nan_mismatch": nan_mismatch}


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def make_inputs(names, rows=None):
    from memory_bound_fk_b200 import synth
    out = {}
    for n in names:
        t = time.perf_counter()
        out[n] = np.ascontiguousarray(synth.make(n, rows=rows))
        log(f"[bench] generated {n} {out[n].shape} in {time.perf_counter() - t:.1f}s")
    return out


# ---------------------------------------------------------------- our arm

class L2Cleaner:
    """Leaves the L2 holding nothing of the timed work: a read-only pass (a
    sum) over a buffer of 4x the L2 size, so that every dirty line left by
    earlier kernels is written back and evicted before the timed launch,
    whose own time then excludes other kernels' write-backs."""

    def __init__(self, device, l2_bytes: int):
        import torch
        self.buf = torch.ones(max(4 * l2_bytes, 256 << 20) // 4, dtype=torch.float32, device=device)
        self.out = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self):
        import torch
        torch.sum(self.buf, dim=0, out=self.out)


def time_alone(call, stream, device, reps: int, cleaner) -> list[float]:
    """reps launches of `call`, each after an L2 clean, each timed alone by
    CUDA events on the launching stream (ms)."""
    import torch
    call()
    ts = []
    for _ in range(reps):
        cleaner()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        torch.cuda.synchronize(device)
        ts.append(a.elapsed_time(b))
    return ts


# Workloads timed one by one with the L2 cleaned before each launch: every
# configuration of the pages' workloads, the small report-only ones too.
ALONE = ["cfg1_gelu", "cfg1_softmax"] + SUITE


def run_ours(args) -> dict | None:
    import numpy as np
    import torch

    import memory_bound_fk_b200 as fk
    from memory_bound_fk_b200 import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    fk.lib()  # fail loudly if libfk.so is missing
    names = workload_list(args.workload)
    alone_names = [n for n in (ALONE if args.workload == "suite" else names)] if not args.no_alone else []
    all_names = names + [n for n in alone_names if n not in names]
    host = make_inputs(all_names, args.rows)
    shapes = {n: host[n].shape for n in all_names}
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream

    # device buffers, inputs resident in HBM before the timed region
    dev_in, dev_out, call_of, params, keep = {}, {}, {}, {}, []
    for n in all_names:
        w = synth.WORKLOADS[n]
        if w.dtype == "bf16":
            t = torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(host[n])
        dev_in[n] = t.to(device)
        dev_out[n] = torch.empty_like(dev_in[n])
        xp, yp = dev_in[n].data_ptr(), dev_out[n].data_ptr()
        if w.op.startswith("layernorm"):
            gb = [torch.from_numpy(a).to(device) for a in synth.layernorm_params(shapes[n][1], w.seed)]
            keep += gb
            params[n] = (gb[0].data_ptr(), gb[1].data_ptr())
        call_of[n] = (lambda w=w, xp=xp, yp=yp, shape=shapes[n], pr=params.get(n):
                      launch_workload(fk, w, xp, yp, shape, sh, pr))
    # bytes of each input (rounded down to fk_copy's 16-byte granule; every
    # full-size workload is a multiple of 16 already)
    in_bytes = {n: dev_in[n].numel() * dev_in[n].element_size() // 16 * 16 for n in all_names}
    bytes_step = sum(workload_bytes(synth.WORKLOADS[n], shapes[n]) for n in names)
    elems_step = sum(host[n].size for n in names)

    # Steps whose bytes are fewer than 4x L2 rotate through copies of their
    # buffers, so that no step finds its inputs (or the previous step's
    # outputs) in L2
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = rotation_sets(bytes_step, l2_bytes)
    sets = [({n: dev_in[n] for n in names}, {n: dev_out[n] for n in names})]
    for _ in range(1, nsets):
        sets.append(({n: dev_in[n].clone() for n in names}, {n: torch.empty_like(dev_out[n]) for n in names}))

    def kernel_call(n, xin, yout):
        w = synth.WORKLOADS[n]
        return lambda: launch_workload(fk, w, xin.data_ptr(), yout.data_ptr(), shapes[n], sh, params.get(n))

    def copy_call(n, xin=None, yout=None):
        """fk_copy of a workload's input into its output buffer: the same
        bytes read and written as the fused kernel, nothing computed."""
        xin = dev_in[n] if xin is None else xin
        yout = dev_out[n] if yout is None else yout
        return lambda: fk.fk_copy(xin.data_ptr(), yout.data_ptr(), in_bytes[n], sh)

    calls = [[(n, kernel_call(n, si[n], so[n])) for n in names] for si, so in sets]
    copy_seqs = [[(n, copy_call(n, si[n], so[n])) for n in names] for si, so in sets]

    def step(seq, evs=None):
        for i, (n, call) in enumerate(seq):
            if evs is not None:
                evs[i].record(stream)
            st = call()
            if st != fk.FK_OK:
                raise fk.FkError(st, n)
        if evs is not None:
            evs[len(seq)].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(device)

    def timed_steps(seqs, steps, per_kernel=True):
        """`steps` passes, pass k over seqs[k % len(seqs)], between barriers;
        the total (ms) and, with per_kernel, per entry the event time of
        every pass (the stretch from its launch to the next entry's launch
        on the stream).  Every event recorded between two kernels holds the
        stream for ~2.6 us on this GPU, so the pass that gives the total of
        a measurement has none (per_kernel=False)."""
        n = len(seqs[0])
        events = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)] \
            if per_kernel else [None] * steps
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        start.record(stream)
        for k in range(steps):
            step(seqs[k % len(seqs)], events[k])
        stop.record(stream)
        barrier()
        per = [[evs[i].elapsed_time(evs[i + 1]) for evs in events] for i in range(n)] if per_kernel else None
        return start.elapsed_time(stop), per

    for k in range(max(args.warmup, min(len(calls), 64))):
        step(calls[k % len(calls)])
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    barrier()
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    if sampler:
        sampler.wait_ready()  # its first reading before the timed region
    # the timed region: K steps, events only at its ends
    total_ms, _ = timed_steps(calls, args.steps, per_kernel=False)
    # per-kernel breakdown: K more steps with an event between every two kernels
    ev_total_ms, per_kernel = timed_steps(calls, args.steps)
    clocks = sampler.stop() if sampler else None
    # slowest rank: the totals, then per kernel the sum, median and minimum
    red = max_over_ranks([total_ms, ev_total_ms] + [sum(t) for t in per_kernel]
                         + [statistics.median(t) for t in per_kernel] + [min(t) for t in per_kernel], world, device)
    nk = len(names)
    max_ms, ev_max_ms = red[0], red[1]
    kernel_sum, kernel_med, kernel_min = red[2:2 + nk], red[2 + nk:2 + 2 * nk], red[2 + 2 * nk:]

    # the copy floor of every slot: the same sequence with each kernel
    # replaced by fk_copy of its bytes, so each copy follows the same
    # predecessor traffic as the kernel it stands for
    for k in range(max(1, args.warmup, min(len(copy_seqs), 64))):
        step(copy_seqs[k % len(copy_seqs)])
    copy_total, _ = timed_steps(copy_seqs, args.steps, per_kernel=False)
    _, copy_per = timed_steps(copy_seqs, args.steps)
    red = max_over_ranks([copy_total] + [statistics.median(t) for t in copy_per], world, device)
    copy_total, copy_med = red[0], red[1:]

    # each workload alone, L2 cleaned before every launch
    alone, event_floor = {}, None
    if alone_names:
        cleaner = L2Cleaner(device, torch.cuda.get_device_properties(device).L2_cache_size)
        reps = max(5, min(args.alone_reps, 200))
        # two events around nothing, after the same clean: the floor of an event-timed interval
        event_floor = max_over_ranks([statistics.fmean(time_alone(lambda: None, stream, device, reps, cleaner))],
                                     world, device)[0]
        for n in alone_names:
            def checked(c=call_of[n], n=n):
                st = c()
                if st != fk.FK_OK:
                    raise fk.FkError(st, n)
            tk = time_alone(checked, stream, device, reps, cleaner)
            tc = time_alone(copy_call(n), stream, device, reps, cleaner)
            red = max_over_ranks([statistics.median(tk), min(tk), statistics.median(tc), min(tc),
                                  statistics.fmean(tk), statistics.fmean(tc)], world, device)
            alone[n] = red
        del cleaner

    # copy ceiling for the dominant kernel's bytes: cudaMemcpy D2D and
    # libfk's plain 16-byte copy, same buffers, timed the same way
    dom_i = max(range(len(names)), key=lambda i: kernel_sum[i])
    copy_ceiling = copy_reference(fk, dev_in[names[dom_i]], dev_out[names[dom_i]], stream, device, world)

    # end to end: pinned host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, names, host, dev_in, dev_out, stream, device, world, bytes_step, params)

    # outputs of every workload as the timed kernels write them (the copy
    # floor overwrote them), for the max-error check below
    for n in all_names:
        st = call_of[n]()
        if st != fk.FK_OK:
            raise fk.FkError(st, n)
    torch.cuda.synchronize(device)

    cpu, errors = None, {}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = host_threads()
        f = oracle_sample_plan(all_names, host, args.cpu_budget, threads)
        res = oracle_run(all_names, host, f, threads, keep=True)
        one = oracle_run(all_names, host, f / max(1, threads), 1)
        cpu = {"value": res["bytes"] / res["seconds"] / 1e9, "unit": UNIT, "cores": threads,
               "value_1_thread": one["bytes"] / one["seconds"] / 1e9,
               "per_workload": {n: {"GB_s": round(r["bytes"] / max(r["seconds"], 1e-9) / 1e9, 4),
                                    "GB_s_1_thread": round(one["per_workload"][n]["bytes"]
                                                           / max(one["per_workload"][n]["seconds"], 1e-9) / 1e9, 4),
                                    "elements": r["elements"]}
                                for n, r in res["per_workload"].items()},
               "kind": "oracle",
               "sample": f"leading {100 * f:.3f}% of every workload ({res['elements']} elements, "
                         f"{res['bytes'] / 1e9:.3f} GB algorithmic, {res['seconds']:.1f} s)"}
        # the GPU outputs of the same leading rows against the oracle's
        for n, ref in res["outputs"].items():
            w = synth.WORKLOADS[n]
            got = dev_out[n][:ref.shape[0]]
            got = got.view(torch.int16).cpu().numpy().view(np.uint16) if w.dtype == "bf16" else got.cpu().numpy()
            errors[n] = dict(max_error(got, ref, w.dtype), elements_checked=int(ref.size))

    if rank != 0:
        return None
    peaks = measured_peaks()

    def gbs_of(nbytes, ms):
        return nbytes / (ms * 1e-3) / 1e9

    def plan_of(n):
        w = synth.WORKLOADS[n]
        code = fk.FK_BF16 if w.dtype == "bf16" else fk.FK_F32
        if w.op.startswith("softmax"):
            return fk.fk_softmax_rows_plan(shapes[n][0], shapes[n][1], code).as_dict()
        if w.op.startswith("layernorm"):
            return fk.fk_layernorm_rows_plan(shapes[n][0], shapes[n][1], code).as_dict()
        return {"path": "gelu"}

    kernels = []
    for i, n in enumerate(names):
        w = synth.WORKLOADS[n]
        ms = kernel_sum[i] / args.steps
        nbytes = workload_bytes(w, shapes[n])
        gbs = gbs_of(nbytes, ms)
        plan = plan_of(n)
        kernels.append({"workload": n, "kernel": kernel_name(w, plan), "plan": plan,
                        "shape": list(shapes[n]), "ms": round(ms, 5), "GB_s": round(gbs, 1),
                        "ms_median": round(kernel_med[i], 5), "ms_min": round(kernel_min[i], 5),
                        "GB_s_median": round(gbs_of(nbytes, kernel_med[i]), 1),
                        "elements_per_s": round(host[n].size / (ms * 1e-3), 1),
                        "pct_of_8TBs": round(100 * gbs / SPEC_HBM_GBS, 2),
                        "frac_of_measured_copy": round(gbs / peaks["hbm_gbs"], 4),
                        "copy_floor_same_slot_ms_median": round(copy_med[i], 5),
                        "copy_floor_same_slot_GB_s": round(gbs_of(nbytes, copy_med[i]), 1),
                        "frac_of_copy_floor_same_slot": round(copy_med[i] / kernel_med[i], 4),
                        "bytes_per_launch": nbytes})
    alone_rows = []
    for n in alone_names:
        w = synth.WORKLOADS[n]
        nbytes = workload_bytes(w, shapes[n])
        kmed, kmin, cmed, cmin, kmean, cmean = alone[n]
        alone_rows.append({"workload": n, "kernel": kernel_name(w, plan_of(n)), "shape": list(shapes[n]),
                           "bytes_per_launch": nbytes, "ms_median": round(kmed, 5), "ms_min": round(kmin, 5),
                           "ms_mean": round(kmean, 5), "GB_s_mean": round(gbs_of(nbytes, kmean), 1),
                           "fk_copy_ms_mean": round(cmean, 5), "frac_of_fk_copy_mean": round(cmean / kmean, 4),
                           "GB_s_median": round(gbs_of(nbytes, kmed), 1), "GB_s_best": round(gbs_of(nbytes, kmin), 1),
                           "pct_of_8TBs_median": round(100 * gbs_of(nbytes, kmed) / SPEC_HBM_GBS, 2),
                           "frac_of_measured_peak": round(gbs_of(nbytes, kmed) / peaks["hbm_gbs"], 4),
                           "fk_copy_ms_median": round(cmed, 5), "fk_copy_GB_s_median": round(gbs_of(nbytes, cmed), 1),
                           "frac_of_fk_copy": round(cmed / kmed, 4),
                           "elements_per_s": round(host[n].size / (kmed * 1e-3), 1),
                           "max_error": errors.get(n)})
    for k in kernels:
        k["max_error"] = errors.get(k["workload"])
    dom = max(range(len(names)), key=lambda i: kernel_sum[i])
    dk = kernels[dom]
    traffic, traffic_src = profiled_traffic(names[dom])
    value = aggregate_value(bytes_step, args.steps, world, max_ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload if args.rows is None else f"{args.workload} (leading {args.rows} rows)",
                   "detail": describe(names),
                   "io_dtypes": sorted({synth.WORKLOADS[n].dtype for n in names}),
                   "bytes_per_step_per_gpu": bytes_step, "elements_per_step_per_gpu": elems_step,
                   "l2": (f"inputs larger than L2: {bytes_step // 2 / 1e9:.2f} GB read per step" if nsets == 1 else
                          f"{nsets} rotating buffer sets ({nsets * bytes_step / 1e9:.2f} GB, at least 4x L2): "
                          "no step finds its inputs or the previous step's outputs in L2"),
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "pct_of_8TBs": round(100 * value / world / SPEC_HBM_GBS, 2),
        "elements_per_s": round(elems_step * args.steps * world / (max_ms * 1e-3), 1),
        "kernels": kernels,
        "copy_floor_step": {"ms_per_step": round(copy_total / args.steps, 5),
                            "GB_s": round(aggregate_value(bytes_step, args.steps, world, copy_total), 1),
                            "what": "the same sequence with every kernel replaced by fk_copy of its bytes"},
        "per_kernel_timing": {"how": "a second pass of the same K steps with a CUDA event between every two "
                                     "kernels (the timed region above has events only at its ends)",
                              "ms_per_step_with_events": round(ev_max_ms / args.steps, 5),
                              "event_cost_us": round(1e3 * (ev_max_ms - max_ms) / (args.steps * len(names)), 3)},
        "alone": {"l2": "L2 written back and evicted (read-only pass over 4x L2) before every launch",
                  "event_floor_ms": round(event_floor, 5) if event_floor is not None else None,
                  "timer": "CUDA events tick in steps of about 2 us on this GPU: for launches of tens of us "
                           "the mean over the launches resolves finer than the median",
                  "reps": max(5, min(args.alone_reps, 200)) if alone_names else 0, "workloads": alone_rows},
        "roofline": {"bound": "hbm", "kernel": dk["kernel"], "workload": names[dom],
                     "achieved": dk["GB_s"], "peak": peaks["hbm_gbs"], "unit": UNIT,
                     "frac": round(dk["GB_s"] / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"],
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_bytes_per_launch": dk["bytes_per_launch"],
                     "copy_ceiling": copy_ceiling,
                     "frac_of_copy_ceiling": (round(dk["GB_s"] / copy_ceiling["fk_copy_GB_s"], 4)
                                              if copy_ceiling else None)},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": len(names) * args.steps,
        "clocks": clocks,
    }
    return line


def run_attention(args) -> dict | None:
    """bench.py --workload attn_causal_bf16 | attn_bf16: the tcgen05 attention
    forward, timed as the other workloads (W warm-ups, K steps between
    barriers, CUDA events on the stream, max over ranks), reported in
    algorithmic TFLOP/s (unmasked pairs only) against the measured bf16
    tensor-core peak."""
    import math

    import torch

    import memory_bound_fk_b200 as fk
    from memory_bound_fk_b200 import synth
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    fk.lib()
    n = args.workload
    w = synth.WORKLOADS[n]
    causal = w.op == "attention"
    host = synth.make(n, rows=args.rows)
    _, bh, t, d = host.shape
    scale = 1.0 / math.sqrt(d)
    flops = synth.attention_flops(bh, t, d, causal)
    qkv = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16).to(device)
    o = torch.empty(bh, t, d, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream

    def call(src=qkv, dst=o):
        st = fk.fk_attention_fwd(src[0].data_ptr(), src[1].data_ptr(), src[2].data_ptr(), dst.data_ptr(), bh, t, d,
                                 int(causal), scale, sh)
        if st != fk.FK_OK:
            raise fk.FkError(st, n)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        call()
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    barrier()
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    if sampler:
        sampler.wait_ready()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        call()
    b.record(stream)
    barrier()
    clocks = sampler.stop() if sampler else None
    max_ms = max_over_ranks([a.elapsed_time(b)], world, device)[0]
    tflops = flops * args.steps * world / (max_ms * 1e-3) / 1e12

    # context: torch's fused attention on the same q, k, v and stream, timed
    # the same way right after (rank 0 of a single-GPU run only)
    library = None
    if rank == 0 and world == 1 and not args.no_library:
        library = library_attention(qkv, o, bh, t, d, causal, scale, flops, args.steps, args.warmup, stream, gpu_id)

    # end to end: q, k, v from pinned host memory in, o back out, every step
    e2e = None
    if not args.no_e2e:
        pin_in = torch.empty(qkv.shape, dtype=torch.int16, pin_memory=True)
        pin_in.copy_(torch.from_numpy(host.view(np.int16)))
        pin_out = torch.empty(o.shape, dtype=torch.int16, pin_memory=True)
        steps = max(3, min(args.steps, args.e2e_steps))
        barrier()
        a.record(stream)
        for _ in range(steps):
            qkv.view(torch.int16).copy_(pin_in, non_blocking=True)
            call()
            pin_out.copy_(o.view(torch.int16), non_blocking=True)
        b.record(stream)
        barrier()
        ms_e = max_over_ranks([a.elapsed_time(b)], world, device)[0]
        e2e = {"value": round(flops * steps * world / (ms_e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": pin_in.numel() * 2, "d2h_bytes_per_step": pin_out.numel() * 2,
               "steps": steps, "ms_per_step": round(ms_e / steps, 3)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = host_threads()
        nb = 1
        t0 = time.perf_counter()
        oracle.attention(*(host[i, :nb] for i in range(3)), scale, causal, nthreads=threads)
        dt = time.perf_counter() - t0
        cpu = {"value": synth.attention_flops(nb, t, d, causal) / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
               "kind": "oracle", "sample": f"{nb} of {bh} (batch, head) slices ({dt:.1f} s)"}
    if rank != 0:
        return None
    d_all = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = float(d_all.get("bf16_tflops", 1590.0))
    ms = max_ms / args.steps
    kname = f"attention_fwd_kernel<d={d},causal={int(causal)}>"
    # DRAM bytes of one launch from the ncu capture in profiles/ (q, k, v
    # read, o written: 4 bh t d bf16 values algorithmically; K/V tiles that
    # miss L2 are read again)
    traffic, traffic_src = profiled_traffic(n)
    return {
        "metric": "attention forward TFLOP/s (bf16 in, fp32 accumulate) at 1 B200", "value": round(tflops, 2),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": n, "detail": w.recipe, "bh": bh, "t": t, "d": d, "causal": causal,
                   "algorithmic_flops_per_step": flops,
                   "l2": "q, k, v total %.0f MB; every launch reads them from HBM or L2" % (qkv.numel() * 2 / 1e6),
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "kernels": [{"workload": n, "kernel": kname, "ms": round(ms, 5), "TFLOP_s": round(flops / ms / 1e9, 1)}],
        "roofline": {"bound": "tensor", "kernel": kname, "workload": n, "achieved": round(flops / ms / 1e9, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(flops / ms / 1e9 / peak, 4),
                     "peak_source": "measured (cuBLAS bf16 burst)" if d_all else "fallback",
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_bytes_per_launch": 4 * bh * t * d * 2},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps, "clocks": clocks,
        "library_context": library,
    }


def library_attention(qkv, o, bh, t, d, causal, scale, flops, steps, warmup, stream, gpu_id) -> dict:
    """torch.nn.functional.scaled_dot_product_attention on the same inputs,
    once per backend that runs on this GPU: W warm-ups, then K calls between
    two CUDA events on the same stream, with the SM clocks sampled meanwhile.
    A reference point for the kernel's speed, not part of this library."""
    import torch
    from torch.nn.attention import SDPBackend, sdpa_kernel
    q4, k4, v4 = (qkv[i].view(1, bh, t, d) for i in range(3))
    ours = o.view(1, bh, t, d).float()
    out = {"what": "torch.nn.functional.scaled_dot_product_attention, same q, k, v, scale and mask, timed right "
                   "after the kernel (context only)", "torch": torch.__version__, "backends": {}}
    import contextlib
    # torch's own choice of backend first (what a caller gets by default),
    # then each fused backend forced
    for label, be in (("DEFAULT", None), ("CUDNN_ATTENTION", SDPBackend.CUDNN_ATTENTION),
                      ("FLASH_ATTENTION", SDPBackend.FLASH_ATTENTION)):
        try:
            with (sdpa_kernel(be) if be is not None else contextlib.nullcontext()):
                def call():
                    return torch.nn.functional.scaled_dot_product_attention(q4, k4, v4, is_causal=causal,
                                                                            scale=scale)
                ref = call()
                for _ in range(warmup):
                    call()
                torch.cuda.synchronize()
                sampler = ClockSampler(gpu_id)
                sampler.wait_ready()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(steps):
                    call()
                b.record(stream)
                torch.cuda.synchronize()
                clocks = sampler.stop()
                ms = a.elapsed_time(b) / steps
                out["backends"][label] = {"TFLOP_s": round(flops / ms / 1e9, 1), "ms": round(ms, 5),
                                          "max_abs_diff_vs_this_kernel": float((ref.float() - ours).abs().max()),
                                          "clocks": clocks}
        except RuntimeError as e:
            out["backends"][label] = {"unavailable": str(e).splitlines()[0][:160]}
    return out


def copy_reference(fk, src, dst, stream, device, world, reps: int = 7) -> dict | None:
    """Median time of copying src's bytes into dst with cudaMemcpyAsync
    (torch's copy_) and with libfk's fk_copy: the achievable-bandwidth
    reference of the same byte count (read + write counted)."""
    import torch
    nbytes = src.numel() * src.element_size()
    if nbytes % 16:
        return None
    out = {}
    for label, fn in (("cudaMemcpy", lambda: dst.copy_(src)),
                      ("fk_copy", lambda: fk.fk_copy(src.data_ptr(), dst.data_ptr(), nbytes, stream.cuda_stream))):
        fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(device)
            ts.append(a.elapsed_time(b))
        ms = max_over_ranks([sorted(ts)[len(ts) // 2]], world, device)[0]
        out[f"{label}_GB_s"] = round(2 * nbytes / (ms * 1e-3) / 1e9, 1)
    out["bytes_copied"] = nbytes
    return out


def run_e2e(args, names, host, dev_in, dev_out, stream, device, world, bytes_step, params=None):
    """Same step through the C ABI from pinned host buffers: every step copies
    all inputs host->device and all outputs device->host inside the timed
    region.  Work is split into row chunks (about --e2e-chunk-mb of input
    each) issued round-robin on --e2e-streams streams, so the host->device copy of one
    chunk, the kernel of another and the device->host copy of a third
    overlap (the two copy directions use separate copy engines)."""
    import torch

    import memory_bound_fk_b200 as fk
    from memory_bound_fk_b200 import synth
    pin_in, pin_out = {}, {}
    for n in names:
        a = host[n]
        src = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        pin_in[n] = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
        pin_in[n].copy_(src)
        pin_out[n] = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
    h2d = sum(pin_in[n].numel() * pin_in[n].element_size() for n in names)
    d2h = sum(pin_out[n].numel() * pin_out[n].element_size() for n in names)

    # chunk plan: (workload, first row, row count) -- GELU is split by elements
    chunk_bytes = max(1, args.e2e_chunk_mb) << 20
    chunks = []
    for n in names:
        a = host[n]
        row_bytes = a.itemsize * (a.shape[1] if a.ndim == 2 else 1)
        per = max(1, chunk_bytes // row_bytes)
        if a.ndim == 1:
            per = max(8, per // 8 * 8)  # keep 16-byte chunk boundaries
        elif synth.WORKLOADS[n].op.startswith("softmax_causal"):
            per = max(1, per // a.shape[1]) * a.shape[1]  # whole query blocks per chunk
        for r0 in range(0, a.shape[0], per):
            chunks.append((n, r0, min(per, a.shape[0] - r0)))
    streams = [stream] + [torch.cuda.Stream(device) for _ in range(max(1, args.e2e_streams) - 1)]
    raw_in = {n: (dev_in[n].view(torch.int16) if dev_in[n].dtype == torch.bfloat16 else dev_in[n]) for n in names}
    raw_out = {n: (dev_out[n].view(torch.int16) if dev_out[n].dtype == torch.bfloat16 else dev_out[n]) for n in names}

    def step():
        for i, (n, r0, cnt) in enumerate(chunks):
            s = streams[i % len(streams)]
            w = synth.WORKLOADS[n]
            with torch.cuda.stream(s):
                raw_in[n][r0:r0 + cnt].copy_(pin_in[n][r0:r0 + cnt], non_blocking=True)
                xp = raw_in[n][r0:r0 + cnt].data_ptr()
                yp = raw_out[n][r0:r0 + cnt].data_ptr()
                st = launch_workload(fk, w, xp, yp, (cnt,) + tuple(host[n].shape[1:]), s.cuda_stream,
                                     (params or {}).get(n))
                if st != fk.FK_OK:
                    raise fk.FkError(st, n)
                pin_out[n][r0:r0 + cnt].copy_(raw_out[n][r0:r0 + cnt], non_blocking=True)

    steps = max(3, min(args.steps, args.e2e_steps))
    step()
    torch.cuda.synchronize(device)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for s2 in streams[1:]:
        s2.wait_stream(stream)
    for _ in range(steps):
        step()
    for s2 in streams[1:]:
        stream.wait_stream(s2)
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks([a.elapsed_time(b)], world, device)[0]
    # the copies really brought the results back: spot-check one chunk's bytes
    n0, r0, cnt = chunks[-1]
    assert torch.equal(pin_out[n0][r0:r0 + cnt], raw_out[n0][r0:r0 + cnt].cpu())
    return {"value": round(aggregate_value(bytes_step, steps, world, ms), 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3), "chunks_per_step": len(chunks), "streams": len(streams)}


# ---------------------------------------------------------------- unfused comparison

GELU_C = 0.7978845608028654  # sqrt(2/pi)


def gelu_unfused(x):
    """tanh-GELU as the printed formula, one PyTorch eager op (one kernel,
    one full read and write of a tensor) per step."""
    import torch
    a = torch.pow(x, 3)
    a = a * 0.044715
    a = x + a
    a = a * GELU_C
    a = torch.tanh(a)
    a = 1.0 + a
    a = x * a
    return 0.5 * a


def softmax_unfused(x):
    """'Manual' row softmax: max, subtract, exp, sum, divide as separate ops."""
    import torch
    m = x.max(dim=-1, keepdim=True).values
    z = x - m
    e = torch.exp(z)
    s = e.sum(dim=-1, keepdim=True)
    return e / s


def unfused_traffic_bytes(op: str, tensor_bytes: int) -> int:
    """HBM bytes of the unfused sequences above if no tensor stays in cache:
    every op reads its full-size inputs and writes its full-size output
    (the per-row max and sum are negligible)."""
    if op == "gelu":
        reads, writes = 10, 8   # pow, mul, add(2), mul, tanh, add, mul(2), mul
    else:
        reads, writes = 5, 3    # max, sub, exp, sum, div
    return (reads + writes) * tensor_bytes


def run_unfused(args) -> dict | None:
    """Times the unfused PyTorch sequences against libfk's fused kernels on
    the same device buffers (one GPU; the lecture's 192 MB vs 64 MB claim)."""
    import torch

    import memory_bound_fk_b200 as fk
    from memory_bound_fk_b200 import synth
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    fk.lib()
    names = workload_list(args.workload)
    host = make_inputs(names, args.rows)
    out = []
    for n in names:
        w = synth.WORKLOADS[n]
        if w.op not in ("gelu", "softmax"):
            raise SystemExit(f"--impl unfused covers tanh-GELU and plain softmax workloads, not {n}")
        a = host[n]
        x = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16
             else torch.from_numpy(a)).to(device)
        y = torch.empty_like(x)
        s = torch.cuda.current_stream(device).cuda_stream
        if w.op == "gelu":
            unf = lambda: gelu_unfused(x)  # noqa: E731
            fused = lambda: fk.fk_gelu_tanh(x.data_ptr(), y.data_ptr(), x.numel(), s)  # noqa: E731
        else:
            code = fk.FK_BF16 if w.dtype == "bf16" else fk.FK_F32
            unf = lambda: softmax_unfused(x)  # noqa: E731
            fused = lambda: fk.fk_softmax_rows(x.data_ptr(), y.data_ptr(), x.shape[0], x.shape[1], code, s)  # noqa: E731
        res = {}
        for label, fn in (("unfused", unf), ("fused", fused)):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize(device)
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record()
            for _ in range(args.steps):
                fn()
            ev1.record()
            torch.cuda.synchronize(device)
            res[label] = ev0.elapsed_time(ev1) / args.steps
        tb = a.nbytes
        out.append({"workload": n, "shape": list(a.shape), "dtype": w.dtype,
                    "unfused_ms": round(res["unfused"], 5), "fused_ms": round(res["fused"], 5),
                    "speedup": round(res["unfused"] / res["fused"], 2),
                    "unfused_traffic_model_bytes": unfused_traffic_bytes(w.op, tb),
                    "fused_traffic_bytes": 2 * tb,
                    "traffic_ratio_model": round(unfused_traffic_bytes(w.op, tb) / (2 * tb), 2)})
        del x, y
        torch.cuda.empty_cache()
    tot_u = sum(o["unfused_ms"] for o in out)
    tot_f = sum(o["fused_ms"] for o in out)
    bytes_step = sum(2 * host[n].nbytes for n in names)
    return {"impl": "unfused", "metric": METRIC, "value": round(bytes_step / (tot_u * 1e-3) / 1e9, 1),
            "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_u, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": args.workload, "detail": describe(names),
                       "what": "PyTorch eager, one kernel per formula step, vs libfk's fused kernels"},
            "fused_value": round(bytes_step / (tot_f * 1e-3) / 1e9, 1),
            "speedup_fused_over_unfused": round(tot_u / tot_f, 2), "workloads": out}


# ---------------------------------------------------------------- reference arm

def run_reference(args) -> dict | None:
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    names = workload_list(args.workload)
    host = make_inputs(names, args.rows)
    threads = host_threads()
    per_step = args.reference_budget / max(1, args.steps + args.warmup)
    f = oracle_sample_plan(names, host, per_step, threads)
    for _ in range(args.warmup):
        oracle_run(names, host, f, threads)
    secs, nbytes, elems = 0.0, 0, 0
    for _ in range(args.steps):
        r = oracle_run(names, host, f, threads)
        secs += r["seconds"]
        nbytes += r["bytes"]
        elems += r["elements"]
    value = nbytes / secs / 1e9
    sample = (f"leading {100 * f:.4f}% of every workload per step "
              f"({elems // max(1, args.steps)} elements per step)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload if args.rows is None else f"{args.workload} (leading {args.rows} rows)",
                   "detail": describe(names),
                   "parallelism": "host cores (oracle)"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main

def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference", "unfused"], default="ours",
                   help="ours: libfk kernels; reference: the CPU oracle; unfused: PyTorch "
                        "eager op-by-op sequences timed against libfk (one GPU)")
    p.add_argument("--workload", default="suite",
                   help="suite (default) or one of cfg1_gelu, cfg1_softmax, cfg2_gelu, "
                        "cfg3_softmax, cfg4_softmax, cfg5_softmax, and the operator variants "
                        "cfg2_gelu_erf, gelu_bf16, gelu_erf_bf16, cfg4_causal, cfg4_causal_skip, ln_f32, ln_gelu_bf16, "
                        "attn_causal_bf16, attn_bf16")
    p.add_argument("--rows", type=int, default=None,
                   help="profiling only: leading rows (elements for GELU) of each workload")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--e2e-chunk-mb", type=int, default=64,
                   help="input bytes per pipelined host<->device chunk in the e2e leg")
    p.add_argument("--e2e-streams", type=int, default=2, help="streams the e2e leg's chunks rotate over")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-alone", action="store_true", help="skip the per-workload L2-clean leg")
    p.add_argument("--no-library", action="store_true",
                   help="attention workloads: skip timing torch's scaled_dot_product_attention beside the kernel")
    p.add_argument("--alone-reps", type=int, default=30, help="launches per workload in the L2-clean leg")
    p.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    p.add_argument("--reference-budget", type=float, default=120.0,
                   help="seconds for the whole --impl reference run")
    a = p.parse_args(argv)
    if a.warmup < 3 and a.impl != "reference" and a.steps > 10:
        p.error("--warmup must be at least 3 for a reported measurement")
    return a


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        line = run_reference(args)
    elif args.impl == "unfused":
        line = run_unfused(args)
    elif args.workload in ("attn_causal_bf16", "attn_bf16"):
        line = run_attention(args)
    else:
        line = run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    if args.impl in ("ours",) and dist_env()[1] > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
