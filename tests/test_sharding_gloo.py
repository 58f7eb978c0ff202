"""Multi-process host logic on CPU (gloo, world sizes 2 and 4): matrix
ownership, the flat reduce-scatter / owner step / all-gather exchange of a
sharded step, its bucketed form (with the gradient reduction in fp32 as an
option, and each owner's EMA of its matrices), and the benchmark's
max-over-ranks timing.  The per-rank compute is
the fp64 oracle here; on GPUs it is the library's step."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from muon_optimizer_step_02_b200 import sharding, workloads as wl


def test_partition_is_balanced_and_complete():
    shapes = wl.workload(2).shapes
    for world in (1, 2, 4, 8):
        owner = sharding.partition_matrices(shapes, world)
        assert len(owner) == len(shapes)
        assert set(owner) <= set(range(world))
        loads = sharding.rank_loads(shapes, owner, world)
        total = sum(loads)
        biggest = max(sharding.matrix_cost(r, c, 5) for r, c in shapes)
        # LPT bound: max load <= total/world + largest item
        assert max(loads) <= total / world + biggest + 1e-6
        assert owner == sharding.partition_matrices(shapes, world)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_flat_layout_is_owner_ordered_and_aligned():
    shapes = wl.workload(2).shapes
    for world in (1, 2, 8):
        L = sharding.ShardLayout(shapes, world)
        assert L.owner == sharding.partition_matrices(shapes, world)
        spans = []
        for i, (r, c) in enumerate(shapes):
            o = L.owner[i]
            assert o * L.seg <= L.offset[i] and L.offset[i] + r * c <= (o + 1) * L.seg
            assert L.offset[i] % 8 == 0
            spans.append((L.offset[i], L.offset[i] + r * c))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))   # no overlap
        assert L.numel() == world * L.seg


SHARES = {2: [0.25, 0.75], 4: [0.125, 0.25, 0.25, 0.375]}
EMA_D = 0.9965


def _flat_worker(rank, world, port, q):
    import oracle.muon_oracle as mo
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        shapes = [(48, 32), (32, 48), (40, 40), (16, 64), (64, 16), (24, 24), (8, 100)]
        h = wl.Hyper(momentum=0.9, lr=0.05, weight_decay=0.1)
        coeffs = [wl.FIXED_QUINTIC] * 3
        w = wl.custom(shapes, h, coeffs, grad_std=1.0, wid=401)
        L = sharding.ShardLayout(shapes, world, 3)
        W_flat = torch.zeros(L.numel(), dtype=torch.float64)
        for i, v in enumerate(L.views(W_flat)):
            v.copy_(torch.from_numpy(wl.weight(w, i).astype(np.float64)))
        M_seg = torch.zeros(L.seg, dtype=torch.float64)
        G_seg = torch.zeros(L.seg, dtype=torch.float64)
        E_seg = torch.zeros(L.seg, dtype=torch.float64)
        for j, v in zip(L.mine[rank], L.local_views(E_seg, rank)):
            v.copy_(torch.from_numpy(wl.weight(w, j).astype(np.float64)))
        hyp = mo.MuonHyper(momentum=h.momentum, lr=h.lr, weight_decay=h.weight_decay)

        def step_fn(Wv, Mv, Gv):
            for a, m, g in zip(Wv, Mv, Gv):
                Wn, Mn, _ = mo.muon_step(a.numpy(), m.numpy(), g.numpy(), hyp, coeffs, 1.0)
                a.copy_(torch.from_numpy(Wn))
                m.copy_(torch.from_numpy(Mn))

        def ema_fn(Ev, Wv):
            for e, a in zip(Ev, Wv):
                e.copy_(torch.from_numpy(mo.ema_update(e.numpy(), a.numpy(), EMA_D)))

        for step in range(2):
            G_flat = torch.zeros(L.numel(), dtype=torch.float64)
            # dyadic shares: the reduce-scatter sums them back to g exactly
            share = SHARES[world][rank]
            for i, v in enumerate(L.views(G_flat)):
                g = wl.bf16_bits_to_f32(wl.grad_bits(w, i, step)).astype(np.float64)
                v.copy_(torch.from_numpy(g * share))
            sharding.sharded_step_flat(L, W_flat, M_seg, G_flat, G_seg, rank, step_fn,
                                       E_seg=E_seg, ema_fn=ema_fn)
        t = sharding.max_over_ranks(1.0 + rank)
        E = {j: v.numpy().copy() for j, v in zip(L.mine[rank], L.local_views(E_seg, rank))}
        q.put((rank, [v.numpy().copy() for v in L.views(W_flat)], t, E))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_flat_sharded_step_matches_single_process(world):
    import oracle.muon_oracle as mo
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_flat_worker, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shapes = [(48, 32), (32, 48), (40, 40), (16, 64), (64, 16), (24, 24), (8, 100)]
    h = wl.Hyper(momentum=0.9, lr=0.05, weight_decay=0.1)
    coeffs = [wl.FIXED_QUINTIC] * 3
    w = wl.custom(shapes, h, coeffs, grad_std=1.0, wid=401)
    hyp = mo.MuonHyper(momentum=h.momentum, lr=h.lr, weight_decay=h.weight_decay)
    W = [wl.weight(w, i).astype(np.float64) for i in range(len(shapes))]
    M = [np.zeros_like(x) for x in W]
    E = [x.copy() for x in W]
    for step in range(2):
        for i in range(len(shapes)):
            G = wl.bf16_bits_to_f32(wl.grad_bits(w, i, step)).astype(np.float64)
            W[i], M[i], _ = mo.muon_step(W[i], M[i], G, hyp, coeffs, 1.0)
            E[i] = mo.ema_update(E[i], W[i], EMA_D)
    owned = set()
    for rank, Ws, t, Er in out:
        assert t == float(world)           # max over ranks of 1.0 + rank
        for a, b in zip(Ws, W):
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
        # each rank's average covers exactly the matrices it owns
        for j, e in Er.items():
            np.testing.assert_allclose(e, E[j], rtol=1e-12, atol=1e-14)
        assert not owned & set(Er)
        owned |= set(Er)
    assert owned == set(range(len(shapes)))


SHAPES_B = [(48, 32), (32, 48), (40, 40), (16, 64), (64, 16), (24, 24), (8, 100),
            (56, 24), (24, 56)]


def _bucket_worker(rank, world, port, q, n_buckets, fp32_reduce):
    import oracle.muon_oracle as mo
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        h = wl.Hyper(momentum=0.9, lr=0.05, weight_decay=0.1)
        coeffs = [wl.FIXED_QUINTIC] * 3
        w = wl.custom(SHAPES_B, h, coeffs, grad_std=1.0, wid=402)
        BL = sharding.BucketedLayout(SHAPES_B, world, n_buckets, 3)
        gdt = torch.float32 if fp32_reduce else torch.float64
        bufs = [sharding.BucketBuffers.allocate(L, torch.float64, gdt, torch.float64,
                                                with_ema=True)
                for L in BL.layouts]
        for bk, L, bf in zip(BL.buckets, BL.layouts, bufs):
            for j, v in enumerate(L.views(bf.W_flat)):
                v.copy_(torch.from_numpy(wl.weight(w, bk[j]).astype(np.float64)))
            for j, v in zip(L.mine[rank], L.local_views(bf.E_seg, rank)):
                v.copy_(torch.from_numpy(wl.weight(w, bk[j]).astype(np.float64)))
        hyp = mo.MuonHyper(momentum=h.momentum, lr=h.lr, weight_decay=h.weight_decay)

        def step_fn(Wv, Mv, Gv):
            for a, m, g in zip(Wv, Mv, Gv):
                Wn, Mn, _ = mo.muon_step(a.numpy(), m.numpy(), g.numpy(), hyp, coeffs, 1.0)
                a.copy_(torch.from_numpy(Wn))
                m.copy_(torch.from_numpy(Mn))

        def ema_fn(Ev, Wv):
            for e, a in zip(Ev, Wv):
                e.copy_(torch.from_numpy(mo.ema_update(e.numpy(), a.numpy(), EMA_D)))

        def to_bf16_values(dst, src):
            # the library rounds the fp32 sum to bf16; the fp64 step reads it
            dst.copy_(src.to(torch.bfloat16).to(torch.float64))

        share = SHARES[world][rank]
        for step in range(2):
            for bk, L, bf in zip(BL.buckets, BL.layouts, bufs):
                bf.G_flat.zero_()
                for j, v in enumerate(L.views(bf.G_flat)):
                    g = wl.bf16_bits_to_f32(wl.grad_bits(w, bk[j], step)).astype(np.float64)
                    v.copy_(torch.from_numpy(g * share))
            sharding.sharded_step_bucketed(BL, bufs, rank, [step_fn] * n_buckets,
                                           to_step_dtype=to_bf16_values if fp32_reduce
                                           else None, ema_fns=[ema_fn] * n_buckets)
        W = [None] * len(SHAPES_B)
        E = {}
        for bk, L, bf in zip(BL.buckets, BL.layouts, bufs):
            for j, v in enumerate(L.views(bf.W_flat)):
                W[bk[j]] = v.numpy().copy()
            for j, v in zip(L.mine[rank], L.local_views(bf.E_seg, rank)):
                E[bk[j]] = v.numpy().copy()
        q.put((rank, W, E))
    finally:
        dist.destroy_process_group()


def test_bucketed_layout_covers_every_matrix_once():
    shapes = wl.workload(2).shapes
    for world in (1, 2, 8):
        for nb in (1, 2, 3, 11, 66):
            BL = sharding.BucketedLayout(shapes, world, nb)
            assert len(BL.buckets) == nb
            flat = [i for bk in BL.buckets for i in bk]
            assert flat == list(range(len(shapes)))      # consecutive, in order
            assert all(bk for bk in BL.buckets)
    with pytest.raises(ValueError):
        sharding.BucketedLayout(shapes, 2, 0)


@pytest.mark.parametrize("world,n_buckets,fp32_reduce",
                         [(2, 2, False), (2, 3, True), (4, 3, False), (4, 2, True)])
def test_bucketed_sharded_step_matches_single_process(world, n_buckets, fp32_reduce):
    import oracle.muon_oracle as mo
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bucket_worker,
                         args=(r, world, port, q, n_buckets, fp32_reduce))
             for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    h = wl.Hyper(momentum=0.9, lr=0.05, weight_decay=0.1)
    coeffs = [wl.FIXED_QUINTIC] * 3
    w = wl.custom(SHAPES_B, h, coeffs, grad_std=1.0, wid=402)
    hyp = mo.MuonHyper(momentum=h.momentum, lr=h.lr, weight_decay=h.weight_decay)
    W = [wl.weight(w, i).astype(np.float64) for i in range(len(SHAPES_B))]
    M = [np.zeros_like(x) for x in W]
    E = [x.copy() for x in W]
    for step in range(2):
        for i in range(len(SHAPES_B)):
            G = wl.bf16_bits_to_f32(wl.grad_bits(w, i, step)).astype(np.float64)
            W[i], M[i], _ = mo.muon_step(W[i], M[i], G, hyp, coeffs, 1.0)
            E[i] = mo.ema_update(E[i], W[i], EMA_D)
    owned = set()
    for rank, Ws, Er in out:
        for a, b in zip(Ws, W):
            # dyadic shares of bf16 values sum exactly in fp32 and in fp64
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
        for j, e in Er.items():
            np.testing.assert_allclose(e, E[j], rtol=1e-12, atol=1e-14)
        assert not owned & set(Er)
        owned |= set(Er)
    assert owned == set(range(len(SHAPES_B)))
