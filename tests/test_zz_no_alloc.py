"""muon_step_batched_noalloc: the entry point for callers that cannot
allocate device memory (a framework that owns all device memory and gives a
plug-in only inputs and outputs, or a loop that forbids cudaMalloc after
start-up).  It runs the same kernels on the same work lists as
muon_step_batched, so over consecutive calls its outputs must equal the
planned step's bit for bit, and both must match the fp64 oracle; it must
allocate nothing; and a bounded wait that runs out must be readable through
muon_noalloc_error_async.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest

import oracle.muon_oracle as mo
from gpu_harness import TOL_STATE, oracle_hyper, rel_fro, tol_o
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(shapes, seed, wid=300):
    import torch
    w = wl.custom(shapes, wl.workload(2).hyper, [wl.FIXED_QUINTIC] * 5,
                  wid=wid)
    W = [torch.from_numpy(wl.weight(w, i, seed)).cuda()
         for i in range(w.n_mats)]
    G = [[torch.from_numpy(wl.grad_bits(w, i, step, seed).view(np.int16))
          .cuda().view(torch.bfloat16) for i in range(w.n_mats)]
         for step in range(2)]
    return w, W, G


def _check_against_oracle(w, W0, M0, G, W1, M1, O1, scales):
    """One step of the fp64 oracle from the pre-step state (W0, M0, G) and
    the library's post-step state (W1, M1) and update O1, compared at the
    tolerances of the parity tests."""
    import torch
    hyp = oracle_hyper(w.hyper)
    for i, shape in enumerate(w.shapes):
        bits = G[i].cpu().view(torch.int16).numpy().view(np.uint16)
        g = wl.bf16_bits_to_f32(bits).astype(np.float64)
        Wr, Mr, Or = mo.muon_step(W0[i], M0[i], g, hyp, w.coeffs, scales[i])
        o1 = O1[i].cpu().numpy().astype(np.float64)
        assert rel_fro(o1, Or) <= tol_o(shape), f"matrix {i}: O"
        assert rel_fro(M1[i].cpu().numpy(), Mr) <= TOL_STATE, f"matrix {i}: M"
        w_given = mo.decoupled_update(W0[i], o1, hyp.lr, hyp.weight_decay,
                                      scales[i])
        assert rel_fro(W1[i].cpu().numpy(), w_given) <= TOL_STATE, \
            f"matrix {i}: W given O"


def test_noalloc_equals_planned_step_and_oracle_on_two_calls():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    # one layer of the 11L x 512d model plus two ragged matrices
    shapes = wl.gpt_layer_shapes(512, 8, 4, 64) + [(300, 200), (7, 13)]
    w, W, G = _inputs(shapes, seed=11)
    scales = wl.update_scales(w)
    # the planned path: plan + caller workspace
    W_ref = [x.clone() for x in W]
    M_ref = [torch.zeros_like(x) for x in W]
    O_ref = [torch.empty_like(x) for x in W]
    plan = B.MuonPlan(shapes, 5)
    ws = plan.alloc_workspace()
    # the allocation-free path on its own copies
    W_na = [x.clone() for x in W]
    M_na = [torch.zeros_like(x) for x in W]
    O_na = [torch.empty_like(x) for x in W]
    word = torch.full((1,), 7, dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()
    for step in range(2):
        W0 = [x.cpu().numpy().astype(np.float64) for x in W_na]
        M0 = [x.cpu().numpy().astype(np.float64) for x in M_na]
        plan.step(W_ref, M_ref, G[step], w.hyper, w.coeffs, ws,
                  update_scales=scales, update_out=O_ref)
        torch.cuda.synchronize()
        # process-local evidence that the call allocates nothing: the
        # library's own device allocations and torch's allocator
        lib_allocs = B.device_allocation_count()
        torch_bytes = torch.cuda.memory_allocated()
        B.muon_step_batched_noalloc(W_na, M_na, G[step], w.hyper, w.coeffs,
                                    update_scales=scales, update_out=O_na)
        B.noalloc_error_async(word)
        torch.cuda.synchronize()
        assert B.device_allocation_count() == lib_allocs
        assert torch.cuda.memory_allocated() == torch_bytes
        assert int(word[0]) == 0
        assert plan.last_error() == 0
        # same kernels, same work lists: bit for bit
        for i in range(len(shapes)):
            assert torch.equal(O_na[i], O_ref[i]), f"step {step} matrix {i}: O"
            assert torch.equal(M_na[i], M_ref[i]), f"step {step} matrix {i}: M"
            assert torch.equal(W_na[i], W_ref[i]), f"step {step} matrix {i}: W"
        _check_against_oracle(w, W0, M0, G[step], W_na, M_na, O_na, scales)
    plan.close()


def test_noalloc_reports_a_bounded_wait_that_ran_out():
    """The test hook makes the tensor-core kernel's first stage never arrive,
    so its bounded wait runs out (about a second): the array's error word is
    set and muon_noalloc_error_async reads it without synchronising.  The next
    call clears it and computes normally."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    shapes = [(256, 512), (512, 256)]
    w, W, G = _inputs(shapes, seed=12, wid=301)
    scales = wl.update_scales(w)
    word = torch.zeros(1, dtype=torch.int32).pin_memory()
    M = [torch.zeros_like(x) for x in W]
    B.noalloc_set_fault(1)
    try:
        B.muon_step_batched_noalloc([x.clone() for x in W], M, G[0], w.hyper,
                                    w.coeffs, update_scales=scales)
        B.noalloc_error_async(word)
        torch.cuda.current_stream().synchronize()
        assert int(word[0]) != 0
    finally:
        B.noalloc_set_fault(0)
    # a clean call on fresh state: the word is cleared, the result is right
    W1 = [x.clone() for x in W]
    M1 = [torch.zeros_like(x) for x in W]
    O1 = [torch.empty_like(x) for x in W]
    W0 = [x.cpu().numpy().astype(np.float64) for x in W1]
    M0 = [np.zeros(s) for s in shapes]
    B.muon_step_batched_noalloc(W1, M1, G[0], w.hyper, w.coeffs,
                                update_scales=scales, update_out=O1)
    word[0] = 7
    B.noalloc_error_async(word)
    torch.cuda.current_stream().synchronize()
    assert int(word[0]) == 0
    _check_against_oracle(w, W0, M0, G[0], W1, M1, O1, scales)


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
