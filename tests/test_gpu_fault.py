"""Failure detection without a GPU fault: the test hook makes the first
stage of the first tile never arrive, so the tensor-core kernel's bounded
wait runs out (about one second), the kernel records the error word, drains
its own copies and MMAs, frees TMEM and returns.  The host must read
MUON_ERR_TIMEOUT, and the same plan must work normally afterwards."""
import numpy as np
import pytest

from gpu_harness import GpuMuon, check_step
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_recoverable():
    import time

    import torch
    from muon_optimizer_step_02_b200 import binding as B
    h = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
    w = wl.custom([(256, 512), (512, 256)], h, [wl.FIXED_QUINTIC] * 5,
                  wid=500)
    g = GpuMuon(w)
    g.plan.set_fault(1)
    t0 = time.time()
    g.step(g.grads(0))
    word = torch.zeros(1, dtype=torch.int32).pin_memory()
    g.plan.error_async(word)              # no synchronisation
    torch.cuda.current_stream().synchronize()
    assert int(word[0]) != 0              # the asynchronous copy saw the error word
    status = g.plan.last_error()          # synchronises the stream
    elapsed = time.time() - t0
    assert status == B.MUON_ERR_TIMEOUT
    assert elapsed < 30.0
    # the error word is cleared by the read
    assert g.plan.last_error() == B.MUON_OK
    # the context and the plan still work: a clean step matches the oracle
    g.plan.set_fault(0)
    torch.cuda.synchronize()
    g2 = GpuMuon(w)
    check_step(g2, 0, [0, 1])
    word[0] = 7
    g2.plan.error_async(word)
    torch.cuda.current_stream().synchronize()
    assert int(word[0]) == 0


def test_refused_launch_is_reported_and_recoverable():
    """Test hook 2: the runtime refuses the tensor-core kernel's launch (more
    shared memory than it was set up for).  The step call returns
    MUON_ERR_CUDA at once, no device error is left behind, and the next step
    on a fresh state matches the oracle."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    h = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
    w = wl.custom([(256, 512), (512, 256)], h, [wl.FIXED_QUINTIC] * 5, wid=501)
    g = GpuMuon(w)
    g.plan.set_fault(2)
    with pytest.raises(B.MuonError) as err:
        g.step(g.grads(0))
    assert err.value.status == B.MUON_ERR_CUDA
    g.plan.set_fault(0)
    torch.cuda.synchronize()
    assert g.plan.last_error() == B.MUON_OK
    g2 = GpuMuon(w)
    check_step(g2, 0, [0, 1])
