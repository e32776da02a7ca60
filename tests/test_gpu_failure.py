"""Failure handling on the GPU without a fault: a bounded device wait that
runs out is reported to the host as SCOPE_ETIMEOUT and leaves the CUDA
context usable.

The wait is the library's own bounded mbarrier wait (the one every
tensor-core kernel uses), made to run out on a barrier that nothing ever
completes, with a limit of about a millisecond."""
import pytest
import torch

import cluster_guided_sparse_b200 as scope
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def tiny_call():
    w = synth.WORKLOADS["tiny"]
    q, k, v = (t.cuda() for t in synth.make_inputs(w))
    params, grid = scope.make_params(w)
    pl = scope.plan(q, k, params, grid)
    o = scope.attn(q, k, v, pl)
    return pl, o


def test_bounded_wait_times_out_and_context_survives():
    pl, _ = tiny_call()
    pl.sync_status()  # a clean call first
    pl.selftest_wait_timeout(2_000_000)
    with pytest.raises(scope.ScopeError) as e:
        pl.sync_status()
    assert e.value.status == 8 and "wait gave up" in str(e.value)
    err = pl.view("error").cpu().tolist()
    assert err[0] & 2 and err[1] == 0x7E  # timeout bit, and where the wait gave up
    # the context still works: a new call runs clean and gives the same output
    pl2, o2 = tiny_call()
    pl2.sync_status()
    pl3, o3 = tiny_call()
    pl3.sync_status()
    assert torch.equal(o2, o3)
