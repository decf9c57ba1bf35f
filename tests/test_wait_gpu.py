"""Failure detection on the cluster paths, without faulting the GPU.

Blocks of a cluster exchange their partial (max, sum) through mbarriers;
each wait is bounded in time and a wait that gives up is counted in a
device word read by fk_wait_timeouts.  The self-test makes a wait run out
(an mbarrier that nothing arrives on) and checks the count; every real
softmax launch must leave the count at zero.
"""
import numpy as np
import pytest

from memory_bound_fk_b200 import synth

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_is_counted_and_the_context_stays_usable(fk, cuda_device):
    import torch
    fk.fk_wait_timeouts(reset=True)
    s = torch.cuda.current_stream()
    assert fk.fk_wait_selftest(2000, s.cuda_stream) == fk.FK_OK   # 2 ms limit
    torch.cuda.synchronize()
    assert fk.fk_wait_timeouts(reset=True) == 32                    # one per thread
    assert fk.fk_wait_timeouts() == 0
    # the context is still healthy: a cluster softmax runs and is exact
    x = torch.from_numpy(synth.softmax_input(4, 131072, "f32", seed=1)).cuda()
    y = fk.softmax_rows(x)
    torch.cuda.synchronize()
    assert abs(float(y.double().sum(dim=1).sub(1).abs().max())) < 1e-5
    assert fk.fk_wait_timeouts() == 0


def test_cluster_launches_never_give_up(fk, cuda_device):
    import torch
    fk.fk_wait_timeouts(reset=True)
    for cols, plan in [(131072, None), (600000, None),
                       (4096, fk.make_plan(fk.FK_PATH_CLUSTER, threads=128, cluster=16, vpt=4)),
                       (50000, fk.make_plan(fk.FK_PATH_TWOPHASE, cluster=16))]:
        x = torch.from_numpy(synth.softmax_input(64, cols, "f32", seed=cols)).cuda()
        fk.softmax_rows(x, plan=plan)
    torch.cuda.synchronize()
    assert fk.fk_wait_timeouts() == 0
