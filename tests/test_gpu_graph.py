"""The step as the benchmark times it: one CUDA graph holding a Muon step and
the EMA, captured after one uncaptured call and replayed, gives the same
weights, momenta, updates and averages as eager calls, bit for bit; and a
step whose buffers changed since the last call refuses to be captured (its
device table would need a host-to-device copy) instead of capturing stale
pointers."""
import pytest

from gpu_harness import GpuMuon
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
Q5 = [wl.FIXED_QUINTIC] * 5
SHAPES = [(512, 512), (256, 512), (2048, 512), (512, 2048), (100, 72)]


def _ema_state(g):
    E = [x.clone().view(-1) for x in g.W]
    P = [x.view(-1) for x in g.W]
    return E, P


def test_graph_replay_of_step_and_ema_matches_eager():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.custom(SHAPES, H, Q5, wid=130)
    a, b = GpuMuon(w), GpuMuon(w)
    Ea, Pa = _ema_state(a)
    Eb, Pb = _ema_state(b)
    Ga, Gb = a.grads(0), b.grads(0)
    run_a = a.plan.bind(a.W, a.M, Ga, w.hyper, w.coeffs, a.ws,
                        update_scales=a.scales, update_out=a.O)
    ema_a = B.ema_bind(Ea, Pa, 0.99)
    run_b = b.plan.bind(b.W, b.M, Gb, w.hyper, w.coeffs, b.ws,
                        update_scales=b.scales, update_out=b.O)
    ema_b = B.ema_bind(Eb, Pb, 0.99)
    for t in range(4):
        for dst, src in zip(Ga, a.grads(t)):
            dst.copy_(src)
        run_a()
        ema_a()
    run_b()              # uncaptured: uploads the plan's table
    ema_b()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            run_b()
            ema_b()
    torch.cuda.current_stream().wait_stream(side)
    for t in range(1, 4):
        for dst, src in zip(Gb, b.grads(t)):
            dst.copy_(src)
        graph.replay()
    torch.cuda.synchronize()
    assert a.plan.last_error() == 0 and b.plan.last_error() == 0
    for i in range(w.n_mats):
        assert torch.equal(a.W[i], b.W[i]), f"matrix {i}: W"
        assert torch.equal(a.M[i], b.M[i]), f"matrix {i}: M"
        assert torch.equal(a.O[i], b.O[i]), f"matrix {i}: O"
        assert torch.equal(Ea[i], Eb[i]), f"matrix {i}: EMA"
    del graph


def test_capture_refused_when_buffers_changed():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.custom([(128, 192)], H, Q5, wid=131)
    g = GpuMuon(w)
    G = g.grads(0)
    g.plan.step(g.W, g.M, G, w.hyper, w.coeffs, g.ws, update_scales=g.scales)
    torch.cuda.synchronize()
    W2 = [x.clone() for x in g.W]        # new weight buffers: the table changes
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    status = None
    with torch.cuda.stream(side):
        try:
            with torch.cuda.graph(graph, stream=side):
                try:
                    g.plan.step(W2, g.M, G, w.hyper, w.coeffs, g.ws,
                                update_scales=g.scales)
                except B.MuonError as e:
                    status = e.status
        except RuntimeError:
            pass                          # an empty capture may be rejected by torch
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert status == B.MUON_ERR_UNSUPPORTED
    del graph
    # the same call outside a capture then uploads the table and updates the
    # new buffers, not the old ones
    W_old = [x.clone() for x in g.W]
    W2_before = [x.clone() for x in W2]
    g.plan.step(W2, g.M, G, w.hyper, w.coeffs, g.ws, update_scales=g.scales)
    torch.cuda.synchronize()
    assert g.plan.last_error() == 0
    assert torch.equal(g.W[0], W_old[0])
    assert not torch.equal(W2[0], W2_before[0])
