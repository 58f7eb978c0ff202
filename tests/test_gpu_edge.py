"""Edge cases of the CUDA path, through the C ABI: ragged and degenerate
shapes, zero rows, step counts 0..5, switches off, determinism, guard
canaries around every output, and host-side error codes."""
import ctypes

import numpy as np
import pytest

import oracle.muon_oracle as mo
from gpu_harness import GpuMuon, TOL_O, TOL_STATE, check_step, oracle_hyper, rel_fro
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
Q5 = [wl.FIXED_QUINTIC] * 5

RAGGED = [(1, 1), (1, 64), (64, 1), (1, 300), (300, 1), (7, 13), (13, 7),
          (16, 16), (129, 257), (257, 129), (200, 300), (300, 200),
          (640, 130), (130, 640), (1000, 8), (8, 1000), (384, 384),
          (2100, 100), (100, 2100), (511, 1025)]


@pytest.mark.parametrize("shape", RAGGED, ids=lambda s: f"{s[0]}x{s[1]}")
def test_ragged_shapes(shape):
    w = wl.custom([shape], H, Q5, grad_std=1.0)
    g = GpuMuon(w)
    for step in range(2):
        check_step(g, step, [0], emu_tol=1e-2)


def test_ragged_batch_in_one_plan():
    w = wl.custom(RAGGED, H, Q5, grad_std=1.0, wid=101)
    g = GpuMuon(w)
    for step in range(2):
        check_step(g, step, list(range(w.n_mats)))


# Row lengths that select each prologue variant: one-pass rows spread over 1,
# 2, 4 and 8 warps (cols a multiple of 8, at most 8192), rows too long for it
# (8200, 8-aligned) and unaligned long rows (8201); the transposed write-out
# with a row over two warps.
PROLOGUE_ROWS = [(24, 1000), (40, 3000), (24, 6000), (16, 8192), (9, 8200),
                 (12, 8201), (1100, 1040)]


@pytest.mark.parametrize("shape", PROLOGUE_ROWS, ids=lambda s: f"{s[0]}x{s[1]}")
def test_prologue_row_lengths(shape):
    w = wl.custom([shape], H, Q5, grad_std=1.0, wid=110)
    g = GpuMuon(w)
    for step in range(2):
        check_step(g, step, [0])


def test_prologue_variants_in_one_plan():
    """One-pass and two-pass prologue items in the same step."""
    w = wl.custom(PROLOGUE_ROWS, H, Q5, grad_std=1.0, wid=111)
    g = GpuMuon(w)
    # both prologue kernels and the Newton-Schulz kernel
    assert g.plan.step_launches(5) == 3
    assert GpuMuon(wl.custom([(24, 1000)], H, Q5)).plan.step_launches(5) == 2
    for step in range(2):
        check_step(g, step, list(range(w.n_mats)))


@pytest.mark.parametrize("k", [1, 2, 4, 5])
def test_step_counts(k):
    w = wl.custom([(256, 512), (512, 256), (200, 136)], H, Q5[:k], wid=102)
    g = GpuMuon(w)
    check_step(g, 0, [0, 1, 2], emu_tol=1e-2)


def test_zero_steps_gives_normalised_direction():
    """K = 0: O is the Frobenius-normalised MuonEq-R direction."""
    w = wl.custom([(96, 160), (160, 96), (7, 13)], H, [], wid=103)
    g = GpuMuon(w)
    check_step(g, 0, [0, 1, 2], coeffs=[])


@pytest.mark.parametrize("nesterov,eq_r", [(False, True), (True, False),
                                           (False, False)])
def test_switches(nesterov, eq_r):
    h = wl.Hyper(momentum=0.9, lr=0.05, weight_decay=0.0, nesterov=nesterov,
                 eq_r=eq_r)
    w = wl.custom([(256, 384), (384, 256)], h, Q5, wid=104)
    g = GpuMuon(w)
    for step in range(2):
        check_step(g, step, [0, 1], emu_tol=1e-2)


def test_zero_gradient_rows_stay_zero():
    import torch
    w = wl.custom([(192, 256), (300, 128)], H, Q5, wid=105)
    g = GpuMuon(w)
    G = g.grads(0)
    G[0][5:9] = 0
    G[1][17] = 0
    g.step(G)
    torch.cuda.synchronize()
    assert g.plan.last_error() == 0
    # zero momentum + zero gradient row -> that row of O is exactly zero
    o0 = g.O[0].cpu().numpy()
    assert np.all(o0[5:9] == 0)
    assert np.all(g.O[1].cpu().numpy()[17] == 0)
    assert np.all(np.isfinite(o0))


def test_heavy_tailed_rows():
    w = wl.custom([(512, 1024), (1024, 512)], wl.workload(4).hyper, Q5,
                  heavy_tailed_rows=True, wid=106)
    g = GpuMuon(w)
    for step in range(2):
        check_step(g, step, [0, 1], emu_tol=1e-2)


def test_later_plan_needing_less_staging_leaves_earlier_plan_working():
    """The prologue kernels' dynamic shared memory limit is a per-device
    setting of each kernel, shared by every plan.  A plan created later whose
    transposed items need less staging (here about 1 KB against 33 KB and
    19 KB) must not lower it below what an earlier plan launches with: the
    earlier plan's steps still run and match the oracle."""
    big = wl.custom([(2048, 512), (700, 300)], H, Q5, grad_std=1.0, wid=520)
    g_big = GpuMuon(big)          # one-pass and two-pass transposed items
    small = wl.custom([(64, 16), (40, 12)], H, Q5, grad_std=1.0, wid=521)
    g_small = GpuMuon(small)
    check_step(g_small, 0, [0, 1])
    check_step(g_big, 0, [0, 1])
    check_step(g_small, 1, [0, 1])
    check_step(g_big, 1, [0, 1])


def test_deterministic():
    import torch
    outs = []
    for _ in range(2):
        w = wl.custom([(512, 2048), (300, 200), (256, 512)], H, Q5, wid=107)
        g = GpuMuon(w)
        for step in range(2):
            g.step(g.grads(step))
        torch.cuda.synchronize()
        outs.append([x.cpu().numpy().copy() for x in g.W + g.M + g.O])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_update_out_optional_same_weights():
    import torch
    res = []
    for with_out in (True, False):
        w = wl.custom([(384, 640), (640, 384)], H, Q5, wid=108)
        g = GpuMuon(w, with_out=with_out)
        g.step(g.grads(0))
        torch.cuda.synchronize()
        res.append([x.cpu().numpy() for x in g.W])
    for a, b in zip(*res):
        assert np.array_equal(a, b)


def test_canaries_untouched():
    """Outputs live inside larger buffers filled with a sentinel; nothing
    outside the tensors changes."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    shapes = [(300, 200), (129, 257), (7, 13)]
    w = wl.custom(shapes, H, Q5, wid=109)
    pad = 64
    SENT = 12345.5

    def guarded(n):
        buf = torch.full((n + 2 * pad,), SENT, dtype=torch.float32,
                         device="cuda")
        return buf, buf[pad:pad + n]

    bufs, W, M, O = [], [], [], []
    for i, (r, c) in enumerate(shapes):
        b1, w1 = guarded(r * c)
        w1.copy_(torch.from_numpy(wl.weight(w, i).reshape(-1)))
        b2, m1 = guarded(r * c)
        m1.zero_()
        b3, o1 = guarded(r * c)
        bufs += [b1, b2, b3]
        W.append(w1.view(r, c))
        M.append(m1.view(r, c))
        O.append(o1.view(r, c))
    G = [torch.from_numpy(wl.grad_bits(w, i).view(np.int16)).cuda()
         .view(torch.bfloat16) for i in range(len(shapes))]
    plan = B.MuonPlan(shapes, 5)
    wsb = torch.full((plan.workspace_bytes + 2 * 4096,), 0x5A,
                     dtype=torch.uint8, device="cuda")
    ws = wsb[4096:4096 + plan.workspace_bytes]
    plan.step(W, M, G, H, Q5, ws, update_out=O)
    E_buf, E = guarded(1000)
    E.zero_()
    B.ema_update_batched([E], [W[0].reshape(-1)[:1000]], 0.9)
    torch.cuda.synchronize()
    assert plan.last_error() == 0
    for b in bufs + [E_buf]:
        h = b.cpu().numpy()
        assert np.all(h[:pad] == SENT) and np.all(h[-pad:] == SENT)
    hw = wsb.cpu().numpy()
    assert np.all(hw[:4096] == 0x5A) and np.all(hw[-4096:] == 0x5A)


def test_error_codes():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    shapes = [(64, 96)]
    plan = B.MuonPlan(shapes, 5)
    W = torch.zeros(64, 96, device="cuda")
    M = torch.zeros_like(W)
    G = torch.zeros(64, 96, device="cuda", dtype=torch.bfloat16)
    ws = plan.alloc_workspace()
    # too small workspace
    with pytest.raises(B.MuonError) as e:
        plan.step([W], [M], [G], H, Q5, ws[:16])
    assert e.value.status == B.MUON_ERR_WORKSPACE
    # more steps than the plan allows
    with pytest.raises(B.MuonError) as e:
        plan.step([W], [M], [G], H, Q5 * 2, ws)
    assert e.value.status == B.MUON_ERR_UNSUPPORTED
    # misaligned weight pointer (offset by one float)
    buf = torch.zeros(64 * 96 + 1, device="cuda")
    Wmis = buf[1:].view(64, 96)
    with pytest.raises(B.MuonError) as e:
        plan.step([Wmis], [M], [G], H, Q5, ws)
    assert e.value.status == B.MUON_ERR_ALIGNMENT
    # shape that does not match the plan, through the raw ABI
    L = B.lib()
    mats = (B.muon_matrix_t * 1)(B.muon_matrix_t(W.data_ptr(), M.data_ptr(),
                                                 G.data_ptr(), None, 96, 64,
                                                 1.0))
    hp = B.muon_hyper_t(0.9, 0.02, 0.0, 1e-7, 1e-7, 1, 1)
    co = (ctypes.c_float * 15)(*([3.4445, -4.775, 2.0315] * 5))
    st = L.muon_step_batched(plan.handle, mats, ctypes.byref(hp), co, 5,
                             ws.data_ptr(), ws.numel(), None)
    assert st == B.MUON_ERR_UNSUPPORTED
    # non-finite hyper-parameter
    hp2 = B.muon_hyper_t(float("nan"), 0.02, 0.0, 1e-7, 1e-7, 1, 1)
    mats[0].rows, mats[0].cols = 64, 96
    st = L.muon_step_batched(plan.handle, mats, ctypes.byref(hp2), co, 5,
                             ws.data_ptr(), ws.numel(), None)
    assert st == B.MUON_ERR_INVALID_ARG
    # the plan still works afterwards
    plan.step([W], [M], [G], H, Q5, ws)
    torch.cuda.synchronize()
    assert plan.last_error() == 0


def test_ema_ragged_and_unaligned():
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    rng = np.random.default_rng(3)
    sizes = [0, 1, 3, 4, 5, 17, 1023, 4096, 100003] + [7] * 200
    E, P, ref = [], [], []
    for i, n in enumerate(sizes):
        off = 1 if i % 3 == 1 else 0   # every third tensor 4-byte aligned only
        e = rng.standard_normal(n + off).astype(np.float32)
        p = rng.standard_normal(n + off).astype(np.float32)
        te = torch.from_numpy(e).cuda()[off:]
        tp = torch.from_numpy(p).cuda()[off:]
        E.append(te)
        P.append(tp)
        ref.append(mo.ema_update(e[off:], p[off:], 0.997))
    B.ema_update_batched(E, P, 0.997)
    torch.cuda.synchronize()
    for e, r in zip(E, ref):
        if r.size:
            assert rel_fro(e.cpu().numpy(), r) <= TOL_STATE
