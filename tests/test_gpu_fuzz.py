"""Seeded random cases against the fp64 oracle: random shapes (1..700 rows
and columns, both orientations, aligned and not), random switches and step
counts (the fixed quintic, or in about a third of the cases the committed
4-step minimax table), several matrices per plan, two consecutive steps.  Each update is
compared with the fp64 oracle at max(2e-2, 1.25 x the distance of the
bf16-emulating oracle (the GPU path's rounding points) from fp64), and with
that emulation at 1e-2 where the emulation is within 1.5e-2 of fp64.  Inputs
with m much smaller than n (weights of about 500 x 32 or 50 x 400) are that
sensitive: their emulation lands 1.7e-2 to 2.6e-2 from fp64, and the
iteration amplifies the difference of summation orders as much as the
roundings, so the emulation distance is only reported there.  40 cases by
default; MUONB200_FUZZ_CASES sets another count (MUONB200_FUZZ_SEED0 the
first seed, MUONB200_FUZZ_MAX_DIM the largest row or column count, 700 by
default) for longer runs."""
import os

import numpy as np
import pytest

from gpu_harness import GpuMuon, check_step
from muon_optimizer_step_02_b200 import workloads as wl
from tables import polar_express_k4

pytestmark = pytest.mark.gpu

Q5 = [wl.FIXED_QUINTIC] * 5


MAX_DIM = int(os.environ.get("MUONB200_FUZZ_MAX_DIM", "700"))


def _case(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 5))
    shapes = []
    for _ in range(n):
        r = int(rng.integers(1, MAX_DIM + 1))
        c = int(rng.integers(1, MAX_DIM + 1))
        if rng.random() < 0.5:            # often a multiple of 8 (one-pass rows)
            c = max(8, c // 8 * 8)
        shapes.append((r, c))
    k = int(rng.integers(0, 6))
    h = wl.Hyper(momentum=float(rng.uniform(0.5, 0.99)),
                 lr=float(rng.uniform(0.005, 0.05)),
                 weight_decay=float(rng.uniform(0.0, 0.2)),
                 nesterov=bool(rng.random() < 0.8), eq_r=bool(rng.random() < 0.8))
    # about a third of the cases take the committed 4-step minimax table
    if rng.random() < 0.3:
        return shapes, h, polar_express_k4()[:min(k, 4)]
    return shapes, h, Q5[:k]


N_CASES = int(os.environ.get("MUONB200_FUZZ_CASES", "40"))
SEED0 = int(os.environ.get("MUONB200_FUZZ_SEED0", "0"))


@pytest.mark.parametrize("seed", list(range(SEED0, SEED0 + N_CASES)))
def test_random_case_matches_oracle(seed):
    shapes, h, coeffs = _case(1000 + seed)
    w = wl.custom(shapes, h, coeffs, grad_std=float(10.0 ** (seed % 3 - 2)),
                  wid=600 + seed)
    g = GpuMuon(w)
    for step in range(2):
        check_step(g, step, list(range(w.n_mats)), emu_tol=1e-2, o_tol_from_emu=True)
