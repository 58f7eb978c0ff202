"""Seeded synthetic workloads: matrix shapes, hyper-parameters and inputs.

This module only draws random numbers and lays out shapes.  It holds none of
the optimizer's arithmetic, so both the CUDA path and the fp64 oracle can take
their inputs from it.  Every array is drawn on the host with NumPy's PCG64,
seeded per (workload, matrix, step, tensor kind), so any one matrix can be
regenerated on its own.

Shapes follow the pages' models:
* PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_ 1.0901",
  table "Architecture and training stack", row "Model": 11 layers, 512d,
  8 query heads, 4 KV heads, MLP 4x; row "Parameters": 34,401,372.
* PR #1557 "Record: SP8192 + Improved Parallel Residuals + Muon 0.97 + ...",
  section "Techniques": 11L x 512d, 8H/4KV, MLP 4x, SP8192 vocabulary.
Hyper-parameters: PR #1893 row "Optimizer" (MATRIX_LR=0.022, momentum 0.99)
and row "EMA" (0.9965); PR #1396 table "Techniques Combined" (WD=0.105,
MuonEq-R, Polar Express 4 steps); PR #1557 "Techniques" (Muon 0.97, LR 0.03).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

# The widely used fixed quintic Muon coefficients.  Not printed on the pages;
# used as the default "fixed coefficients" input table (the library treats the
# table purely as input).
FIXED_QUINTIC = (3.4445, -4.7750, 2.0315)


@dataclass(frozen=True)
class Hyper:
    momentum: float
    lr: float
    weight_decay: float
    eps_row: float = 1e-7
    eps_frob: float = 1e-7
    nesterov: bool = True
    eq_r: bool = True


@dataclass
class Workload:
    name: str
    shapes: List[Tuple[int, int]]            # (rows, cols) of every matrix
    hyper: Hyper
    coeffs: List[Tuple[float, float, float]]
    grad_std: float = 1e-3
    weight_std: float = 0.02
    heavy_tailed_rows: bool = False          # per-row scale exp(N(0,1))
    ema_decay: Optional[float] = None
    # Extra (non-matrix) parameter tensors covered by the EMA, as numels.
    ema_extra_numels: List[int] = field(default_factory=list)
    ema_extra_names: List[str] = field(default_factory=list)
    wid: int = 0                              # seed component

    @property
    def n_mats(self) -> int:
        return len(self.shapes)

    def numel(self) -> int:
        return sum(r * c for r, c in self.shapes)

    def ema_numels(self) -> List[int]:
        return [r * c for r, c in self.shapes] + list(self.ema_extra_numels)


def gpt_layer_shapes(d: int, n_q: int, n_kv: int, head_dim: int,
                     mlp_mult: int = 4) -> List[Tuple[int, int]]:
    """Q, K, V, O, MLP up, MLP down of one GPT block in (out, in) layout."""
    q = n_q * head_dim
    kv = n_kv * head_dim
    h = mlp_mult * d
    return [(q, d), (kv, d), (kv, d), (d, q), (h, d), (d, h)]


def default_update_scale(rows: int, cols: int) -> float:
    """Per-matrix update scale input: sqrt(max(1, rows/cols)).  The pages
    print no scale; this is one common choice and only an input."""
    return math.sqrt(max(1.0, rows / cols))


def _cfg1() -> Workload:
    return Workload(
        name="single 128x128 matrix, K=5 fixed quintic",
        shapes=[(128, 128)],
        hyper=Hyper(momentum=0.95, lr=0.02, weight_decay=0.0),
        coeffs=[FIXED_QUINTIC] * 5, grad_std=1.0, wid=1)


def _gpt11_shapes() -> List[Tuple[int, int]]:
    return gpt_layer_shapes(512, 8, 4, 64) * 11


def _cfg2() -> Workload:
    return Workload(
        name="11L x 512d GPT, 66 matrices, K=5 fixed quintic",
        shapes=_gpt11_shapes(),
        hyper=Hyper(momentum=0.99, lr=0.022, weight_decay=0.105),
        coeffs=[FIXED_QUINTIC] * 5, wid=2)


def gpt11_ema_extras() -> Tuple[List[int], List[str]]:
    """Non-matrix parameters of the 11L x 512d model covered by the EMA:
    8192x512 and 4096x512 embedding tables plus 1-D tensors sized to the page's
    34,401,372-parameter residual (118 vectors of 512 and 92 singletons)."""
    numels = [8192 * 512, 4096 * 512] + [512] * 118 + [1] * 92
    names = ["tok_emb", "aux_emb"] + [f"vec{i}" for i in range(118)] + \
        [f"scalar{i}" for i in range(92)]
    return numels, names


def _cfg3(ns_coeffs) -> Workload:
    """The 4-step table is an input (the pages print no coefficients); the
    tests and the benchmark pass the committed minimax table."""
    if ns_coeffs is None or len(ns_coeffs) != 4:
        raise ValueError("the K=4 workload needs its 4-row (a, b, c) table "
                         "as ns_coeffs")
    numels, names = gpt11_ema_extras()
    return Workload(
        name="11L x 512d GPT, 66 matrices, K=4 Polar-Express table + EMA",
        shapes=_gpt11_shapes(),
        hyper=Hyper(momentum=0.97, lr=0.03, weight_decay=0.105),
        coeffs=[tuple(float(v) for v in r) for r in ns_coeffs], ema_decay=0.9965,
        ema_extra_numels=numels, ema_extra_names=names, wid=3)


def _cfg4() -> Workload:
    return Workload(
        name="16L x 1024d GPT, 96 matrices, heavy-tailed gradient rows, K=5",
        shapes=gpt_layer_shapes(1024, 16, 8, 64) * 16,
        hyper=Hyper(momentum=0.99, lr=0.022, weight_decay=0.105),
        coeffs=[FIXED_QUINTIC] * 5, heavy_tailed_rows=True, wid=4)


def _cfg5() -> Workload:
    numels = [8192 * 2048] + [2048] * (24 * 4)
    names = ["tok_emb"] + [f"vec{i}" for i in range(24 * 4)]
    return Workload(
        name="24L x 2048d GPT, 144 matrices, K=5 + EMA",
        shapes=gpt_layer_shapes(2048, 16, 8, 128) * 24,
        hyper=Hyper(momentum=0.99, lr=0.022, weight_decay=0.105),
        coeffs=[FIXED_QUINTIC] * 5, ema_decay=0.9965,
        ema_extra_numels=numels, ema_extra_names=names, wid=5)


def _cfg_bench() -> Workload:
    """The 66-matrix K=5 step plus the EMA over every parameter of the same
    model: one pass over every row of the hot path."""
    numels, names = gpt11_ema_extras()
    w = _cfg2()
    w.name = "11L x 512d GPT: 66-matrix Muon (K=5 fixed quintic) + EMA 0.9965"
    w.ema_decay = 0.9965
    w.ema_extra_numels = numels
    w.ema_extra_names = names
    w.wid = 6
    return w


WORKLOADS = {1: _cfg1, 2: _cfg2, 4: _cfg4, 5: _cfg5, 6: _cfg_bench}


def workload(idx: int, ns_coeffs=None) -> Workload:
    """Workload idx (1-6).  Workload 3 runs a 4-step coefficient table that
    the caller passes as ns_coeffs (rows of (a, b, c))."""
    if idx == 3:
        return _cfg3(ns_coeffs)
    return WORKLOADS[idx]()


# --------------------------------------------------------------------------
# Random inputs
# --------------------------------------------------------------------------

KIND_W, KIND_G, KIND_ROWSCALE, KIND_E, KIND_P, KIND_ADAM = 1, 2, 3, 4, 5, 6


def _rng(seed: int, wid: int, idx: int, step: int, kind: int):
    return np.random.Generator(np.random.PCG64([seed, wid, idx, step, kind]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the 16-bit
    patterns.  Input preparation: the gradients arrive in bf16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def weight(w: Workload, idx: int, seed: int = 1337) -> np.ndarray:
    r, c = w.shapes[idx]
    g = _rng(seed, w.wid, idx, 0, KIND_W)
    return (g.standard_normal((r, c), dtype=np.float32)
            * np.float32(w.weight_std))


def grad_bits(w: Workload, idx: int, step: int = 0,
              seed: int = 1337) -> np.ndarray:
    """bf16 gradient of matrix idx at optimizer step `step` (16-bit patterns,
    rows x cols)."""
    r, c = w.shapes[idx]
    g = _rng(seed, w.wid, idx, step, KIND_G)
    x = g.standard_normal((r, c), dtype=np.float32) * np.float32(w.grad_std)
    if w.heavy_tailed_rows:
        s = _rng(seed, w.wid, idx, step, KIND_ROWSCALE).standard_normal(r)
        x = x * np.exp(s).astype(np.float32)[:, None]
    return f32_to_bf16_bits(x)


def ema_pair(w: Workload, idx: int, seed: int = 1337):
    """(E, P) fp32 arrays for EMA tensor idx (matrix params first, then the
    extra tensors in order)."""
    n = w.ema_numels()[idx]
    e = _rng(seed, w.wid, idx, 0, KIND_E).standard_normal(n, dtype=np.float32)
    p = _rng(seed, w.wid, idx, 0, KIND_P).standard_normal(n, dtype=np.float32)
    return e * np.float32(0.02), p * np.float32(0.02)


def adamw_state(numel: int, idx: int, seed: int = 1337, wid: int = 200):
    """(P, M, V, E) fp32 arrays for non-matrix tensor idx of an AdamW + EMA
    case: P, E ~ N(0, 0.02^2); a running first moment M ~ N(0, 1e-3^2) and
    second moment V = (N(0, 1e-3^2))^2 (non-negative), as after a few steps."""
    r = _rng(seed, wid, idx, 0, KIND_ADAM)
    p = r.standard_normal(numel, dtype=np.float32) * np.float32(0.02)
    m = r.standard_normal(numel, dtype=np.float32) * np.float32(1e-3)
    v = (r.standard_normal(numel, dtype=np.float32) * np.float32(1e-3)) ** 2
    e = r.standard_normal(numel, dtype=np.float32) * np.float32(0.02)
    return p, m, v, e


def adamw_grad(numel: int, idx: int, step: int, seed: int = 1337, wid: int = 200):
    """fp32 gradient of non-matrix tensor idx at a step, N(0, 1e-3^2)."""
    return (_rng(seed, wid, idx, step, KIND_ADAM + 1)
            .standard_normal(numel, dtype=np.float32) * np.float32(1e-3))


def update_scales(w: Workload) -> List[float]:
    return [default_update_scale(r, c) for r, c in w.shapes]


def custom(shapes: Sequence[Tuple[int, int]], hyper: Hyper,
           coeffs, grad_std: float = 1e-3, name: str = "custom",
           wid: int = 100, heavy_tailed_rows: bool = False) -> Workload:
    return Workload(name=name, shapes=list(shapes), hyper=hyper,
                    coeffs=list(coeffs), grad_std=grad_std, wid=wid,
                    heavy_tailed_rows=heavy_tailed_rows)
