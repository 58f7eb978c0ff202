"""Scheduled momentum and learning rate (muon_step_batched_sched): the step
number lives in device memory, the kernels read the ramps' values at it and
the call advances it, so a CUDA graph captured once replays every step.
Checked against the fp64 oracle at the scheduled values of each step, and a
graph replay against eager calls, bit for bit."""
import numpy as np
import pytest

import oracle.muon_oracle as mo
from gpu_harness import (GpuMuon, TOL_STATE, oracle_hyper, rel_fro, tol_o)
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = wl.Hyper(momentum=0.0, lr=0.0, weight_decay=0.1)   # momentum, lr unused
Q5 = [wl.FIXED_QUINTIC] * 5
MU = (0.5, 0.9, 1, 3)        # ramps inside the first steps
LR = (0.05, 0.01, 0, 2)
WARMUP = (0.92, 0.99, 0, 1500)   # the pages' momentum warm-up


def _sched_step(g, G, step_dev, sched):
    g.plan.step(g.W, g.M, G, g.w.hyper, g.w.coeffs, g.ws,
                update_scales=g.scales, update_out=g.O, schedule=sched,
                step_dev=step_dev)


def _check_against_oracle(g, t, W0, M0, gstep, sched):
    hyp = mo.scheduled_hyper(oracle_hyper(g.w.hyper), sched[0], sched[1], t)
    for i, shape in enumerate(g.w.shapes):
        Gh = wl.bf16_bits_to_f32(wl.grad_bits(g.w, i, gstep, g.seed)).astype(np.float64)
        Wr, Mr, Or = mo.muon_step(W0[i], M0[i], Gh, hyp, g.w.coeffs, g.scales[i])
        O1 = g.O[i].cpu().numpy().astype(np.float64)
        assert rel_fro(O1, Or) <= tol_o(shape), f"step {t} matrix {i}: O"
        assert rel_fro(g.M[i].cpu().numpy(), Mr) <= TOL_STATE, f"step {t} matrix {i}: M"
        Wg = mo.decoupled_update(W0[i], O1, hyp.lr, hyp.weight_decay, g.scales[i])
        assert rel_fro(g.W[i].cpu().numpy(), Wg) <= TOL_STATE, f"step {t} matrix {i}: W"


def test_scheduled_steps_follow_the_ramps():
    import torch
    w = wl.custom([(256, 384), (384, 256), (100, 72)], H, Q5, wid=120)
    g = GpuMuon(w)
    step_dev = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(5):
        W0 = [x.cpu().numpy().astype(np.float64) for x in g.W]
        M0 = [x.cpu().numpy().astype(np.float64) for x in g.M]
        _sched_step(g, g.grads(t), step_dev, (MU, LR))
        torch.cuda.synchronize()
        assert g.plan.last_error() == 0
        _check_against_oracle(g, t, W0, M0, t, (MU, LR))
    assert int(step_dev.item()) == 5


def test_schedule_reads_the_device_step():
    """Started at step 1000 of the pages' warm-up (0.92 -> 0.99 over 1500
    steps): the momentum of that step is 0.92 + 0.07 * 2/3."""
    import torch
    w = wl.custom([(192, 256), (320, 128)], H, Q5, wid=121)
    g = GpuMuon(w)
    step_dev = torch.full((1,), 1000, dtype=torch.int32, device="cuda")
    lr = (0.02, 0.02, 0, 0)
    for t in (1000, 1001):
        W0 = [x.cpu().numpy().astype(np.float64) for x in g.W]
        M0 = [x.cpu().numpy().astype(np.float64) for x in g.M]
        _sched_step(g, g.grads(t - 1000), step_dev, (WARMUP, lr))
        torch.cuda.synchronize()
        assert g.plan.last_error() == 0
        _check_against_oracle(g, t, W0, M0, t - 1000, (WARMUP, lr))
    assert int(step_dev.item()) == 1002


def test_graph_replay_matches_eager_calls():
    """One graph captured after a warm call replays steps 1..4 with the
    schedule's values; the states equal those of eager calls bit for bit."""
    import torch
    w = wl.custom([(256, 512), (512, 256), (130, 200)], H, Q5, wid=122)
    a, b = GpuMuon(w), GpuMuon(w)
    sa = torch.zeros(1, dtype=torch.int32, device="cuda")
    sb = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(5):
        _sched_step(a, a.grads(t), sa, (MU, LR))
    Gs = b.grads(0)                      # the graph's gradient buffers
    run = b.plan.bind(b.W, b.M, Gs, w.hyper, w.coeffs, b.ws,
                      update_scales=b.scales, update_out=b.O,
                      schedule=(MU, LR), step_dev=sb)
    run()                                # uncaptured: uploads the tables
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            run()
    torch.cuda.current_stream().wait_stream(side)
    for t in range(1, 5):
        for dst, src in zip(Gs, b.grads(t)):
            dst.copy_(src)
        graph.replay()
    torch.cuda.synchronize()
    assert a.plan.last_error() == 0 and b.plan.last_error() == 0
    assert int(sa.item()) == 5 and int(sb.item()) == 5
    for i in range(w.n_mats):
        assert torch.equal(a.W[i], b.W[i]), f"matrix {i}: W differs"
        assert torch.equal(a.M[i], b.M[i]), f"matrix {i}: M differs"
    del graph


def test_schedule_argument_errors():
    import ctypes
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.custom([(64, 96)], H, Q5, wid=123)
    g = GpuMuon(w)
    step_dev = torch.zeros(2, dtype=torch.int32, device="cuda")
    L = B.lib()
    mats = (B.muon_matrix_t * 1)(B.muon_matrix_t(
        g.W[0].data_ptr(), g.M[0].data_ptr(), g.grads(0)[0].data_ptr(), None,
        64, 96, 1.0))
    hp = B.muon_hyper_t(0.0, 0.0, 0.0, 1e-7, 1e-7, 1, 1)
    co = (ctypes.c_float * 15)(*([3.4445, -4.775, 2.0315] * 5))
    ok = B.make_schedule(MU, LR)
    bad_mu = B.make_schedule((0.5, 1.0, 0, 10), LR)          # momentum 1
    bad_lr = B.make_schedule(MU, (float("inf"), 0.01, 0, 2))
    ws, n = g.ws.data_ptr(), g.ws.numel()
    def call(sch, sp):
        return L.muon_step_batched_sched(g.plan.handle, mats, ctypes.byref(hp),
                                         sch, sp, co, 5, ws, n, None)
    assert call(None, step_dev.data_ptr()) == B.MUON_ERR_INVALID_ARG
    assert call(ctypes.byref(ok), None) == B.MUON_ERR_INVALID_ARG
    assert call(ctypes.byref(bad_mu), step_dev.data_ptr()) == B.MUON_ERR_INVALID_ARG
    assert call(ctypes.byref(bad_lr), step_dev.data_ptr()) == B.MUON_ERR_INVALID_ARG
    assert call(ctypes.byref(ok), step_dev.data_ptr() + 2) == B.MUON_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert int(step_dev[0].item()) == 0          # nothing was enqueued


def test_scheduled_step_without_newton_schulz():
    """K = 0: the finishing kernel takes the scheduled learning rate too."""
    import torch
    w = wl.custom([(96, 160), (160, 96)], H, [], wid=124)
    g = GpuMuon(w)
    step_dev = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(3):
        W0 = [x.cpu().numpy().astype(np.float64) for x in g.W]
        M0 = [x.cpu().numpy().astype(np.float64) for x in g.M]
        _sched_step(g, g.grads(t), step_dev, (MU, LR))
        torch.cuda.synchronize()
        assert g.plan.last_error() == 0
        _check_against_oracle(g, t, W0, M0, t, (MU, LR))
    assert int(step_dev.item()) == 3
