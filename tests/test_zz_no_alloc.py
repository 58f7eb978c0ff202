"""muon_step_batched_noalloc: the entry point for callers that cannot
allocate device memory (a framework that owns all device memory and gives a
plug-in only inputs and outputs, or a loop that forbids cudaMalloc after
start-up).  It must give the same result as muon_step_batched on the same
inputs, over consecutive calls, while allocating nothing.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest

from gpu_harness import TOL_O, TOL_STATE, rel_fro, tol_o
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(shapes, seed):
    import torch
    w = wl.custom(shapes, wl.workload(2).hyper, [wl.FIXED_QUINTIC] * 5,
                  wid=300)
    W = [torch.from_numpy(wl.weight(w, i, seed)).cuda()
         for i in range(w.n_mats)]
    G = [[torch.from_numpy(wl.grad_bits(w, i, step, seed).view(np.int16))
          .cuda().view(torch.bfloat16) for i in range(w.n_mats)]
         for step in range(2)]
    return w, W, G


def test_noalloc_matches_planned_step_on_two_calls():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    # one layer of the 11L x 512d model plus two ragged matrices
    shapes = wl.gpt_layer_shapes(512, 8, 4, 64) + [(300, 200), (7, 13)]
    w, W, G = _inputs(shapes, seed=11)
    scales = wl.update_scales(w)
    # reference path: plan + caller workspace
    W_ref = [x.clone() for x in W]
    M_ref = [torch.zeros_like(x) for x in W]
    O_ref = [torch.empty_like(x) for x in W]
    plan = B.MuonPlan(shapes, 5)
    ws = plan.alloc_workspace()
    # no-allocation path
    W_na = [x.clone() for x in W]
    M_na = [torch.zeros_like(x) for x in W]
    O_na = [torch.empty_like(x) for x in W]
    torch.cuda.synchronize()
    for step in range(2):
        plan.step(W_ref, M_ref, G[step], w.hyper, w.coeffs, ws,
                  update_scales=scales, update_out=O_ref)
        if step == 1:
            torch.cuda.synchronize()
            free_before, _ = torch.cuda.mem_get_info()
        B.muon_step_batched_noalloc(W_na, M_na, G[step], w.hyper, w.coeffs,
                                    update_scales=scales, update_out=O_na)
        torch.cuda.synchronize()
        if step == 1:
            free_after, _ = torch.cuda.mem_get_info()
            # the second call allocates nothing on the device
            assert free_after >= free_before
        assert plan.last_error() == 0
        for i, s in enumerate(shapes):
            assert rel_fro(O_na[i].cpu().numpy(), O_ref[i].cpu().numpy()) <= tol_o(s)
            assert rel_fro(M_na[i].cpu().numpy(), M_ref[i].cpu().numpy()) <= TOL_STATE
            assert rel_fro(W_na[i].cpu().numpy(), W_ref[i].cpu().numpy()) <= TOL_STATE
    plan.close()


def test_noalloc_rejects_what_does_not_fit():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    h = wl.workload(2).hyper
    # a matrix whose working copies exceed the fixed scratch array
    W = [torch.zeros(4096, 4096, device="cuda")]
    M = [torch.zeros_like(W[0])]
    G = [torch.zeros(4096, 4096, device="cuda", dtype=torch.bfloat16)]
    with pytest.raises(B.MuonError) as e:
        B.muon_step_batched_noalloc(W, M, G, h, [wl.FIXED_QUINTIC] * 5)
    assert e.value.status == B.MUON_ERR_WORKSPACE
    # more matrices than the fixed tables hold
    n = B.NOALLOC_MAX_MATS + 1
    Ws = [torch.zeros(16, 16, device="cuda") for _ in range(n)]
    Ms = [torch.zeros_like(x) for x in Ws]
    Gs = [torch.zeros(16, 16, device="cuda", dtype=torch.bfloat16)
          for _ in range(n)]
    with pytest.raises(B.MuonError) as e:
        B.muon_step_batched_noalloc(Ws, Ms, Gs, h, [wl.FIXED_QUINTIC] * 5)
    assert e.value.status == B.MUON_ERR_UNSUPPORTED
