"""The AdamW step of the non-matrix parameters fused with their EMA
(adamw_ema_batched), through the C ABI, against the fp64 oracle: ragged and
unaligned tensors, tensors without an EMA, the host and the device step
count, a captured graph against eager calls, and argument errors."""
import ctypes

import numpy as np
import pytest

import oracle.muon_oracle as mo
from gpu_harness import TOL_STATE, rel_fro
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = mo.AdamWHyper(lr=0.01, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
DECAY = 0.9965
# empty, tails of 1..3 elements, a full tensor, the 11L model's 8192 x 512
# embedding and vectors of 512, and an odd size
SIZES = [0, 1, 3, 5, 4096, 8192 * 512, 512, 512, 1000, 4099]


class State:
    """Device tensors of one case; tensor 3 starts one element into its
    buffers (4-byte but not 16-byte aligned: the scalar path); tensors 2 and
    8 have no EMA."""

    def __init__(self, sizes, seed=1337):
        import torch
        self.sizes = sizes
        self.host = [wl.adamw_state(n, i, seed) for i, n in enumerate(sizes)]
        self.bufs = []
        self.P, self.M, self.V, self.E, self.G = [], [], [], [], []
        for i, (n, (p, m, v, e)) in enumerate(zip(sizes, self.host)):
            off = 1 if i == 3 else 0
            def dev(a):
                b = torch.zeros(n + off, dtype=torch.float32, device="cuda")
                b[off:] = torch.from_numpy(a)
                self.bufs.append(b)
                return b[off:]
            self.P.append(dev(p))
            self.M.append(dev(m))
            self.V.append(dev(v))
            self.E.append(None if i in (2, 8) else dev(e))
            self.G.append(dev(np.zeros(n, np.float32)))

    def set_grads(self, step):
        import torch
        for i, n in enumerate(self.sizes):
            self.G[i].copy_(torch.from_numpy(wl.adamw_grad(n, i, step)))

    def snapshot(self):
        return [tuple(None if x is None else x.cpu().numpy().astype(np.float64)
                      for x in (self.P[i], self.M[i], self.V[i], self.E[i]))
                for i in range(len(self.sizes))]


def _check(st, before, t, gstep):
    after = st.snapshot()
    for i, n in enumerate(st.sizes):
        p0, m0, v0, e0 = before[i]
        g = wl.adamw_grad(n, i, gstep).astype(np.float64)
        if e0 is None:
            pr, mr, vr = mo.adamw_update(p0, g, m0, v0, H, t)
            er = None
        else:
            pr, mr, vr, er = mo.adamw_ema(p0, g, m0, v0, e0, H, t, DECAY)
        p1, m1, v1, e1 = after[i]
        for got, ref, what in ((p1, pr, "P"), (m1, mr, "M"), (v1, vr, "V"), (e1, er, "E")):
            if ref is None:
                continue
            assert rel_fro(got, ref) <= TOL_STATE, f"tensor {i} ({n}) step {t}: {what}"


def test_adamw_ema_matches_oracle_host_step():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    st = State(SIZES)
    run = B.adamw_ema_bind(st.P, st.G, st.M, st.V, st.E, H, DECAY)
    for t in (1, 2, 3):
        st.set_grads(t)
        before = st.snapshot()
        run(step_now=t)
        torch.cuda.synchronize()
        _check(st, before, t, t)


def test_device_step_counter_and_graph_replay():
    """Steps counted on the device give the host-step results bit for bit,
    eagerly and from a graph captured once; the counter ends at the number of
    steps taken."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    a, b, c = State(SIZES), State(SIZES), State(SIZES)
    run_a = B.adamw_ema_bind(a.P, a.G, a.M, a.V, a.E, H, DECAY)
    sb = torch.zeros(1, dtype=torch.int32, device="cuda")
    sc = torch.zeros(1, dtype=torch.int32, device="cuda")
    run_b = B.adamw_ema_bind(b.P, b.G, b.M, b.V, b.E, H, DECAY, step_dev=sb)
    run_c = B.adamw_ema_bind(c.P, c.G, c.M, c.V, c.E, H, DECAY, step_dev=sc)
    for t in range(1, 5):
        a.set_grads(t)
        run_a(step_now=t)
        b.set_grads(t)
        run_b()
    c.set_grads(1)
    run_c()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            run_c()
    torch.cuda.current_stream().wait_stream(side)
    for t in range(2, 5):
        c.set_grads(t)
        graph.replay()
    torch.cuda.synchronize()
    assert int(sb.item()) == 4 and int(sc.item()) == 4
    for i in range(len(SIZES)):
        for x, y, z in ((a.P[i], b.P[i], c.P[i]), (a.M[i], b.M[i], c.M[i]),
                        (a.V[i], b.V[i], c.V[i])):
            assert torch.equal(x, y) and torch.equal(x, z), f"tensor {i}"
        if a.E[i] is not None:
            assert torch.equal(a.E[i], b.E[i]) and torch.equal(a.E[i], c.E[i])
    del graph


def test_many_tensors_take_several_launches():
    """More tensors than one launch's segment table (480): the call splits
    them over launches; every tensor still matches the oracle."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    sizes = [(7 * i) % 37 for i in range(500)]
    st = State(sizes, seed=99)
    run = B.adamw_ema_bind(st.P, st.G, st.M, st.V, st.E, H, DECAY)
    st.set_grads(1)
    before = st.snapshot()
    run(step_now=1)
    torch.cuda.synchronize()
    _check(st, before, 1, 1)


def test_adamw_launch_count():
    from muon_optimizer_step_02_b200 import binding as B
    assert B.adamw_ema_launches(len(SIZES)) == 1
    assert B.adamw_ema_launches(len(SIZES), True) == 2
    assert B.adamw_ema_launches(481) == 2
    assert B.adamw_ema_launches(212) == 1     # the 11L model's non-matrix tensors


def test_adamw_argument_errors():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    L = B.lib()
    x = torch.zeros(9, dtype=torch.float32, device="cuda")
    ptr = x.data_ptr()
    good = (B.adamw_tensor_t * 1)(B.adamw_tensor_t(ptr, ptr + 4, ptr + 8, ptr + 12,
                                                   None, 1))
    h = B.adamw_hyper_t(0.01, 0.9, 0.95, 1e-8, 0.1)
    bad_beta = B.adamw_hyper_t(0.01, 1.0, 0.95, 1e-8, 0.1)
    neg_eps = B.adamw_hyper_t(0.01, 0.9, 0.95, -1.0, 0.1)
    mis = (B.adamw_tensor_t * 1)(B.adamw_tensor_t(ptr + 2, ptr + 4, ptr + 8, ptr + 12,
                                                  None, 1))
    neg = (B.adamw_tensor_t * 1)(B.adamw_tensor_t(ptr, ptr + 4, ptr + 8, ptr + 12,
                                                  None, -1))
    null = (B.adamw_tensor_t * 1)(B.adamw_tensor_t(ptr, None, ptr + 8, ptr + 12,
                                                   None, 4))
    E = B.MUON_ERR_INVALID_ARG
    assert L.adamw_ema_batched(good, 1, ctypes.byref(h), 1, None, 0.9, None) == 0
    assert L.adamw_ema_batched(good, 1, ctypes.byref(h), 0, None, 0.9, None) == E
    assert L.adamw_ema_batched(good, 1, ctypes.byref(bad_beta), 1, None, 0.9, None) == E
    assert L.adamw_ema_batched(good, 1, ctypes.byref(neg_eps), 1, None, 0.9, None) == E
    assert L.adamw_ema_batched(good, 1, None, 1, None, 0.9, None) == E
    assert L.adamw_ema_batched(neg, 1, ctypes.byref(h), 1, None, 0.9, None) == E
    assert L.adamw_ema_batched(null, 1, ctypes.byref(h), 1, None, 0.9, None) == E
    assert L.adamw_ema_batched(mis, 1, ctypes.byref(h), 1, None, 0.9, None) == \
        B.MUON_ERR_ALIGNMENT
    assert L.adamw_ema_batched(good, 1, ctypes.byref(h), 1, ptr + 2, 0.9, None) == \
        B.MUON_ERR_ALIGNMENT
    assert L.adamw_ema_batched(None, 0, ctypes.byref(h), 1, None, 0.9, None) == 0
    torch.cuda.synchronize()
