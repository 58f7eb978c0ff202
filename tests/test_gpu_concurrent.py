"""The step next to other work on the GPU.

The Newton-Schulz kernel is persistent: its clusters wait (bounded, about a
second) on items owned by other clusters, so it needs all of its clusters to
become resident eventually.  Here a side stream keeps the GPU busy with a
bounded burst of cuBLAS GEMMs (a few to a few tens of milliseconds) issued
just before the step, so the step's clusters become resident only as the
GEMM blocks retire.  The step must still finish with no device error (no
spurious MUON_ERR_TIMEOUT: the burst is far shorter than the wait limit) and
match the fp64 oracle; the GEMM results must be right too."""
import numpy as np
import pytest

import oracle.muon_oracle as mo
from gpu_harness import GpuMuon, TOL_STATE, oracle_hyper, rel_fro, tol_o
from muon_optimizer_step_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu

H = wl.Hyper(momentum=0.95, lr=0.02, weight_decay=0.1)
Q5 = [wl.FIXED_QUINTIC] * 5


@pytest.mark.parametrize("gemms", [4, 30])
def test_step_while_a_side_stream_holds_the_sms(gemms):
    import torch
    shapes = wl.gpt_layer_shapes(512, 8, 4, 64) * 2
    w = wl.custom(shapes, H, Q5, wid=800 + gemms)
    g = GpuMuon(w)
    hyp = oracle_hyper(w.hyper)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    a = torch.randn(8192, 8192, device="cuda", generator=gen, dtype=torch.bfloat16)
    want = (a[:64].float() @ a[:, :64].float())
    side = torch.cuda.Stream()
    for step in range(2):
        W0 = [x.cpu().numpy().astype(np.float64) for x in g.W]
        M0 = [x.cpu().numpy().astype(np.float64) for x in g.M]
        G = g.grads(step)
        torch.cuda.synchronize()
        outs = []
        with torch.cuda.stream(side):
            for _ in range(gemms):
                outs.append(a @ a)
        g.step(G)           # enqueued while the GEMMs occupy the GPU
        torch.cuda.synchronize()
        assert g.plan.last_error() == 0
        for i in range(len(shapes)):
            gi = wl.bf16_bits_to_f32(wl.grad_bits(w, i, step)).astype(np.float64)
            _, Mr, Or = mo.muon_step(W0[i], M0[i], gi, hyp, w.coeffs, g.scales[i])
            O1 = g.O[i].cpu().numpy().astype(np.float64)
            assert rel_fro(O1, Or) <= tol_o(shapes[i]), f"matrix {i}: O"
            assert rel_fro(g.M[i].cpu().numpy(), Mr) <= TOL_STATE, f"matrix {i}: M"
            w_given = mo.decoupled_update(W0[i], O1, hyp.lr, hyp.weight_decay, g.scales[i])
            assert rel_fro(g.W[i].cpu().numpy(), w_given) <= TOL_STATE, f"matrix {i}: W"
        for c in outs[:: max(1, gemms // 3)]:
            err = (c[:64, :64].float() - want).abs().max().item()
            assert err <= 0.02 * want.abs().max().item()
