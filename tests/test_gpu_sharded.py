"""The sharded step over NCCL with one rank on one GPU, checked against the
fp64 oracle: the flat form (one reduce-scatter of the gradients, the
owner's library step on views of the flat buffers, one all-gather of the
weights) and the bucketed form (reduce-scatters on a communication stream
overlapping the buckets' steps, all-gathers overlapping the later steps),
with the gradients reduced in bf16 or in fp32 (rounded to bf16 by the
library before the step).  With one rank the reduction is the identity, so
the owner's W', M' and O must match the oracle on the same gradients, and
the owner's EMA of its matrices (the library's EMA kernel on views of its
segment) the average of the updated weights.
Several ranks are covered on the CPU by the gloo tests; this checks the CUDA
and NCCL plumbing, the streams and the buffer views the library steps."""
import socket

import numpy as np
import pytest

import oracle.muon_oracle as mo
from gpu_harness import TOL_STATE, oracle_hyper, rel_fro, tol_o
from muon_optimizer_step_02_b200 import sharding
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
Q5 = [wl.FIXED_QUINTIC] * 5
SHAPES = wl.gpt_layer_shapes(512, 8, 4, 64) * 2 + [(300, 200)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def nccl_group():
    import torch.distributed as dist
    dist.init_process_group("nccl", rank=0, world_size=1,
                            init_method=f"tcp://127.0.0.1:{_free_port()}")
    yield
    dist.destroy_process_group()


def _oracle_check(w, i, W0, M0, step, W1, M1, O1):
    hyp = oracle_hyper(w.hyper)
    g = wl.bf16_bits_to_f32(wl.grad_bits(w, i, step)).astype(np.float64)
    _, Mr, Or = mo.muon_step(W0, M0, g, hyp, w.coeffs, wl.update_scales(w)[i])
    o1 = O1.cpu().numpy().astype(np.float64)
    assert rel_fro(o1, Or) <= tol_o(w.shapes[i]), f"matrix {i}: O"
    assert rel_fro(M1.cpu().numpy(), Mr) <= TOL_STATE, f"matrix {i}: M"
    w_given = mo.decoupled_update(W0, o1, hyp.lr, hyp.weight_decay, wl.update_scales(w)[i])
    assert rel_fro(W1.cpu().numpy(), w_given) <= TOL_STATE, f"matrix {i}: W"


EMA_D = 0.9965


def _ema_check(E0, W1, E1, what):
    """E1 (GPU) against E0 d + (1 - d) W1 in fp64 on the GPU's own W1."""
    e_ref = mo.ema_update(E0, W1.cpu().numpy().astype(np.float64), EMA_D)
    assert rel_fro(E1.cpu().numpy(), e_ref) <= TOL_STATE, f"{what}: EMA"


def _ema_fn(B):
    def ema_fn(Ev, Wv):
        B.ema_update_batched([e.view(-1) for e in Ev], [x.view(-1) for x in Wv], EMA_D)
    return ema_fn


def test_flat_sharded_step_single_rank_nccl(nccl_group):
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.custom(SHAPES, H, Q5, grad_std=1.0, wid=150)
    L = sharding.ShardLayout(SHAPES, 1)
    W_flat = torch.zeros(L.numel(), dtype=torch.float32, device="cuda")
    for i, v in enumerate(L.views(W_flat)):
        v.copy_(torch.from_numpy(wl.weight(w, i)))
    M_seg = torch.zeros(L.seg, dtype=torch.float32, device="cuda")
    O_seg = torch.zeros(L.seg, dtype=torch.float32, device="cuda")
    E_seg = W_flat[:L.seg].clone()          # one rank owns every matrix
    G_flat = torch.zeros(L.numel(), dtype=torch.bfloat16, device="cuda")
    G_seg = torch.zeros(L.seg, dtype=torch.bfloat16, device="cuda")
    mine = L.mine[0]
    plan = B.MuonPlan([SHAPES[i] for i in mine], 5)
    ws = plan.alloc_workspace()
    scales = [wl.update_scales(w)[i] for i in mine]

    def step_fn(Wv, Mv, Gv):
        plan.step(Wv, Mv, Gv, H, Q5, ws, update_scales=scales,
                  update_out=L.local_views(O_seg, 0))

    for step in range(2):
        W0 = [v.cpu().numpy().astype(np.float64) for v in L.views(W_flat)]
        M0 = [v.cpu().numpy().astype(np.float64) for v in L.local_views(M_seg, 0)]
        E0 = [v.cpu().numpy().astype(np.float64) for v in L.local_views(E_seg, 0)]
        for i, v in enumerate(L.views(G_flat)):
            v.copy_(torch.from_numpy(wl.grad_bits(w, i, step).view(np.int16))
                    .view(torch.bfloat16))
        sharding.sharded_step_flat(L, W_flat, M_seg, G_flat, G_seg, 0, step_fn,
                                   E_seg=E_seg, ema_fn=_ema_fn(B))
        torch.cuda.synchronize()
        assert plan.last_error() == 0
        Wv, Mv, Ov = L.views(W_flat), L.local_views(M_seg, 0), L.local_views(O_seg, 0)
        Ev = L.local_views(E_seg, 0)
        for j, i in enumerate(mine):
            _oracle_check(w, i, W0[i], M0[j], step, Wv[i], Mv[j], Ov[j])
            _ema_check(E0[j], Wv[i], Ev[j], f"matrix {i}")
    plan.close()


@pytest.mark.parametrize("fp32_reduce", [False, True])
def test_bucketed_sharded_step_single_rank_nccl(nccl_group, fp32_reduce):
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.custom(SHAPES, H, Q5, grad_std=1.0, wid=151)
    BL = sharding.BucketedLayout(SHAPES, 1, 3)
    gdt = torch.float32 if fp32_reduce else torch.bfloat16
    bufs = [sharding.BucketBuffers.allocate(L, torch.float32, gdt, torch.bfloat16, "cuda",
                                            with_ema=True)
            for L in BL.layouts]
    O = [torch.zeros(L.seg, dtype=torch.float32, device="cuda") for L in BL.layouts]
    plans, steps = [], []
    for b, (bk, L, bf) in enumerate(zip(BL.buckets, BL.layouts, bufs)):
        for j, v in enumerate(L.views(bf.W_flat)):
            v.copy_(torch.from_numpy(wl.weight(w, bk[j])))
        bf.E_seg.copy_(bf.W_flat[:L.seg])   # one rank owns every matrix
        mine = [bk[j] for j in L.mine[0]]
        plan = B.MuonPlan([SHAPES[i] for i in mine], 5)
        ws = plan.alloc_workspace()
        scales = [wl.update_scales(w)[i] for i in mine]
        plans.append(plan)

        def step_fn(Wv, Mv, Gv, plan=plan, ws=ws, scales=scales, Ob=O[b], L=L):
            plan.step(Wv, Mv, Gv, H, Q5, ws, update_scales=scales,
                      update_out=L.local_views(Ob, 0))
        steps.append(step_fn)
    comm = torch.cuda.Stream()
    for step in range(2):
        W0, M0, E0 = {}, {}, {}
        for bk, L, bf in zip(BL.buckets, BL.layouts, bufs):
            for j, v in enumerate(L.views(bf.W_flat)):
                W0[bk[j]] = v.cpu().numpy().astype(np.float64)
            for j, v in zip(L.mine[0], L.local_views(bf.M_seg, 0)):
                M0[bk[j]] = v.cpu().numpy().astype(np.float64)
            for j, v in zip(L.mine[0], L.local_views(bf.E_seg, 0)):
                E0[bk[j]] = v.cpu().numpy().astype(np.float64)
            for j, v in enumerate(L.views(bf.G_flat)):
                g = torch.from_numpy(wl.grad_bits(w, bk[j], step).view(np.int16)) \
                    .view(torch.bfloat16)
                v.copy_(g.to(gdt))
        sharding.sharded_step_bucketed(BL, bufs, 0, steps, comm_stream=comm,
                                       to_step_dtype=B.f32_to_bf16 if fp32_reduce else None,
                                       ema_fns=[_ema_fn(B)] * len(bufs))
        torch.cuda.synchronize()
        for plan in plans:
            assert plan.last_error() == 0
        for b, (bk, L, bf) in enumerate(zip(BL.buckets, BL.layouts, bufs)):
            Wv = L.views(bf.W_flat)
            for j, Mj, Oj, Ej in zip(L.mine[0], L.local_views(bf.M_seg, 0),
                                     L.local_views(O[b], 0), L.local_views(bf.E_seg, 0)):
                i = bk[j]
                _oracle_check(w, i, W0[i], M0[i], step, Wv[j], Mj, Oj)
                _ema_check(E0[i], Wv[j], Ej, f"matrix {i}")
    for plan in plans:
        plan.close()


def test_f32_to_bf16_rounds_to_nearest_even():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    g = torch.Generator().manual_seed(3)
    for n in (0, 1, 7, 8, 1000, 4096 + 5):
        src = torch.randn(n, generator=g) * 3.0
        if n >= 8:
            # exact ties: the half-way point between two bf16 values
            src[:4] = torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0])
        want = src.to(torch.bfloat16)
        for off in (0, 1):                      # 16-byte aligned and not
            s = torch.zeros(n + off, device="cuda")
            d = torch.zeros(n + off, dtype=torch.bfloat16, device="cuda")
            s[off:].copy_(src)
            B.f32_to_bf16(d[off:], s[off:])
            torch.cuda.synchronize()
            assert torch.equal(d[off:].cpu(), want)
