"""The flat sharded step (one reduce-scatter of the gradients, the owner's
library step on views of the flat buffers, one all-gather of the weights)
over NCCL with one rank on one GPU: the same kernels on the same inputs as
a plain step, so the weights and momenta must agree bit for bit.  (Several
ranks are covered on the CPU by the gloo tests; this checks the CUDA and
NCCL plumbing and the buffer views the library steps.)"""
import socket

import numpy as np
import pytest

from muon_optimizer_step_02_b200 import sharding
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
Q5 = [wl.FIXED_QUINTIC] * 5
SHAPES = wl.gpt_layer_shapes(512, 8, 4, 64) + [(300, 200)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_flat_sharded_step_single_rank_nccl():
    import torch
    import torch.distributed as dist
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.custom(SHAPES, H, Q5, grad_std=1.0, wid=150)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            init_method=f"tcp://127.0.0.1:{_free_port()}")
    try:
        L = sharding.ShardLayout(SHAPES, 1)
        W_flat = torch.zeros(L.numel(), dtype=torch.float32, device="cuda")
        for i, v in enumerate(L.views(W_flat)):
            v.copy_(torch.from_numpy(wl.weight(w, i)))
        M_seg = torch.zeros(L.seg, dtype=torch.float32, device="cuda")
        G_flat = torch.zeros(L.numel(), dtype=torch.bfloat16, device="cuda")
        G_seg = torch.zeros(L.seg, dtype=torch.bfloat16, device="cuda")
        plan = B.MuonPlan([SHAPES[i] for i in L.mine[0]], 5)
        ws = plan.alloc_workspace()

        def step_fn(Wv, Mv, Gv):
            plan.step(Wv, Mv, Gv, H, Q5, ws)

        # the plain step on separate buffers
        ref = B.MuonPlan(SHAPES, 5)
        ws_ref = ref.alloc_workspace()
        W_ref = [torch.from_numpy(wl.weight(w, i)).cuda() for i in range(len(SHAPES))]
        M_ref = [torch.zeros_like(x) for x in W_ref]
        for step in range(2):
            G = [torch.from_numpy(wl.grad_bits(w, i, step).view(np.int16)).cuda()
                 .view(torch.bfloat16) for i in range(len(SHAPES))]
            for v, g in zip(L.views(G_flat), G):
                v.copy_(g)
            sharding.sharded_step_flat(L, W_flat, M_seg, G_flat, G_seg, 0, step_fn)
            ref.step(W_ref, M_ref, G, H, Q5, ws_ref)
        torch.cuda.synchronize()
        assert plan.last_error() == 0 and ref.last_error() == 0
        Mv = L.local_views(M_seg, 0)
        order = L.mine[0]
        for i, v in enumerate(L.views(W_flat)):
            assert torch.equal(v, W_ref[i]), f"matrix {i}: W"
        for j, i in enumerate(order):
            assert torch.equal(Mv[j], M_ref[i]), f"matrix {i}: M"
    finally:
        dist.destroy_process_group()
