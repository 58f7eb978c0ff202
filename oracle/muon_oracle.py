"""fp64 CPU oracle for the batched Muon optimizer step and the batched EMA pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code with the CUDA library and imports nothing from the package.

Sources (web pages of the parameter-golf competition):

* PR #1584 "Record: Improved Parallel Residuals + Systems Optimization",
  section "Summary": the step being accelerated is a fused Muon kernel plus a
  batched EMA.
* PR #1396 "Record: Combined 3-Layer Recurrence + Parallel Residuals + Polar
  Express + Brotli", table "Techniques Combined": rows "Polar Express
  Newton-Schulz" (4 minimax-optimal steps), "MuonEq-R" (row-norm before NS),
  "WD=0.105"; section "Reproduction" (MUON_WD=0.105 MUON_EQ_R=1).
* PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_ 1.0901",
  table "Architecture and training stack": rows "Optimizer" (Muon on matrix
  params, MATRIX_LR=0.022, momentum 0.99) and "EMA" (EMA_DECAY=0.9965).
* PR #1557 "Record: SP8192 + Improved Parallel Residuals + Muon 0.97 + ...",
  section "Techniques": Muon 0.97 (row-normalized), Matrix LR 0.03, EMA 0.997.

The pages name these steps but print no formula for any of them.  The
per-matrix algorithm below is the method's stated definition, taken in order:

  1. momentum        M' = mu*M + G
  2. Nesterov        U  = G + mu*M'          (U = M' when nesterov is off)
  3. MuonEq-R        U_i <- U_i / (||U_i||_2 + eps_r)   for each stored row i
  4. orientation     X = U^T if rows > cols else U      (X is m x n, m <= n)
  5. Frobenius       X <- X / (||X||_F + eps_f)
  6. Newton-Schulz   for k in 0..K-1:  A = X X^T;  B = b_k A + c_k A A;
                                        X <- a_k X + B X
  7. orientation     O = X^T if transposed else X
  8. update          W' = W (1 - lr*wd) - lr*scale*O
  9. EMA             E' = d*E + (1-d)*P

Readings taken where the pages are silent:
the "sum" Nesterov form; epsilons added to the norm, not inside the square
root; the row norm taken over rows of the stored (out x in) weight before any
transpose; transpose iff rows > cols; weight decay applied to the
pre-update weight; the coefficient table and the per-matrix update scale
are inputs.

Every function here is pinned by tests in tests/test_oracle_pins.py against
closed forms, invariants, library routines (LAPACK SVD) and exact rational
arithmetic on tiny inputs.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import numpy as np

__all__ = [
    "MuonHyper",
    "bf16_round",
    "nesterov_momentum",
    "muon_eq_r",
    "orient",
    "frobenius_normalize",
    "newton_schulz",
    "decoupled_update",
    "muon_step",
    "muon_step_batched",
    "ema_update",
    "ema_update_batched",
    "linear_ramp",
    "scheduled_hyper",
    "AdamWHyper",
    "adamw_update",
    "adamw_ema",
    "ns_flops",
]


@dataclass(frozen=True)
class MuonHyper:
    """Per-call scalars of one Muon step.

    momentum, lr, weight_decay: the pages' Muon settings (e.g. 0.99 / 0.022 /
    0.105 in PR #1893 table "Architecture and training stack", row
    "Optimizer", and PR #1396 table "Techniques Combined", row "WD=0.105").
    eps_row, eps_frob: added to the row norm and the Frobenius norm.
    nesterov, eq_r: switches for the look-ahead form and MuonEq-R.
    """

    momentum: float = 0.95
    lr: float = 0.02
    weight_decay: float = 0.0
    eps_row: float = 1e-7
    eps_frob: float = 1e-7
    nesterov: bool = True
    eq_r: bool = True


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned
    as fp64.  Goes through fp32 first, which is exact for the values the
    emulated path stores (they are fp32-representable products of fp32 math)
    up to one extra rounding; the emulation mode is a diagnostic, the
    spec comparison always uses the unrounded fp64 path."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    out = u.astype(np.uint32).view(np.float32).astype(np.float64)
    # NaN/Inf pass through unchanged.
    bad = ~np.isfinite(f)
    if np.any(bad):
        out[bad] = f[bad]
    return out


def nesterov_momentum(M: np.ndarray, G: np.ndarray, mu: float,
                      nesterov: bool = True):
    """Steps 1-2: momentum accumulation and the Nesterov look-ahead.

    Pages: PR #1893 table "Architecture and training stack", row "Optimizer"
    (momentum 0.99); PR #1557 section "Techniques" (Muon 0.97).  The pages
    give mu but not the update rule; the "sum" form is taken:
    M' = mu*M + G and U = G + mu*M'.
    Returns (M', U) in fp64.
    """
    M = np.asarray(M, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M_new = mu * M + G
    U = G + mu * M_new if nesterov else M_new.copy()
    return M_new, U


def muon_eq_r(U: np.ndarray, eps_row: float) -> np.ndarray:
    """Step 3: MuonEq-R, each row of the stored rows x cols matrix divided by
    its Euclidean norm plus eps_row.

    Pages: PR #1396 table "Techniques Combined", row "MuonEq-R" (row-norm
    before NS); PR #1557 section "Techniques" ("row-normalized").
    A zero row stays zero.
    """
    U = np.asarray(U, dtype=np.float64)
    r = np.sqrt(np.sum(U * U, axis=1))
    return U / (r + eps_row)[:, None]


def orient(U: np.ndarray) -> tuple[np.ndarray, bool]:
    """Step 4: the working matrix X is the short-wide orientation of U
    (m = min(rows, cols) rows).  Transposed iff rows > cols; square matrices
    are not transposed.  Returns (X, transposed)."""
    rows, cols = U.shape
    if rows > cols:
        return U.T.copy(), True
    return U.copy(), False


def frobenius_normalize(X: np.ndarray, eps_frob: float) -> np.ndarray:
    """Step 5: X / (||X||_F + eps_frob), so every singular value is <= 1
    before the Newton-Schulz iteration."""
    X = np.asarray(X, dtype=np.float64)
    return X / (np.sqrt(np.sum(X * X)) + eps_frob)


def newton_schulz(X: np.ndarray, coeffs: Sequence[Sequence[float]],
                  round_fn: Optional[Callable[[np.ndarray], np.ndarray]] = None
                  ) -> np.ndarray:
    """Step 6: K quintic Newton-Schulz steps with per-step coefficients.

    Pages: PR #1396 table "Techniques Combined", row "Polar Express
    Newton-Schulz" (4 minimax-optimal steps).  The coefficient table is an
    input, so a fixed-coefficient schedule and a Polar-Express-style table are
    the same code path.  Each step is A = X X^T, B = b A + c A A, X <- a X + B X.

    round_fn (diagnostic emulation only): applied where a bf16 path stores
    values.  Such a path stores A, then the matrix a I + B (so that
    X <- (a I + B) X is one product; in exact arithmetic this is the same
    step), then the intermediate X; the last X is not rounded.
    """
    X = np.asarray(X, dtype=np.float64)
    K = len(coeffs)
    for k, (a, b, c) in enumerate(coeffs):
        A = X @ X.T
        if round_fn is None:
            B = b * A + c * (A @ A)
            X = a * X + B @ X
        else:
            A = round_fn(A)
            Bp = round_fn(a * np.eye(A.shape[0]) + b * A + c * (A @ A))
            X = Bp @ X
            if k + 1 < K:
                X = round_fn(X)
    return X


def decoupled_update(W: np.ndarray, O: np.ndarray, lr: float, wd: float,
                     scale: float) -> np.ndarray:
    """Step 8: decoupled weight decay on the pre-update weight, then the
    scaled orthogonalised update: W' = W (1 - lr*wd) - lr*scale*O.

    Pages: PR #1396 table "Techniques Combined", row "WD=0.105"; PR #1893
    table "Architecture and training stack", row "Optimizer" (MATRIX_LR)."""
    W = np.asarray(W, dtype=np.float64)
    O = np.asarray(O, dtype=np.float64)
    return W * (1.0 - lr * wd) - (lr * scale) * O


def muon_step(W: np.ndarray, M: np.ndarray, G: np.ndarray, hyper: MuonHyper,
              coeffs: Sequence[Sequence[float]], scale: float,
              emulate_bf16: bool = False):
    """One Muon step for one rows x cols matrix (steps 1-8 in order).

    Returns (W', M', O) in fp64.  With emulate_bf16 the working matrix is
    rounded to bf16 where a bf16 tensor-core path stores it (the row-normalised
    X, A, B and intermediate X); this mode exists to tighten GPU diagnostics,
    the fp64 mode is the reference.
    """
    M_new, U = nesterov_momentum(M, G, hyper.momentum, hyper.nesterov)
    if hyper.eq_r:
        U = muon_eq_r(U, hyper.eps_row)
    X, transposed = orient(U)
    if emulate_bf16:
        # The bf16 path stores the row-normalised matrix and folds the
        # Frobenius scale (computed from the unrounded values) into its first
        # Newton-Schulz step.
        s = 1.0 / (np.sqrt(np.sum(X * X)) + hyper.eps_frob)
        X = s * bf16_round(X)
        O = newton_schulz(X, coeffs, round_fn=bf16_round)
    else:
        X = frobenius_normalize(X, hyper.eps_frob)
        O = newton_schulz(X, coeffs)
    if transposed:
        O = O.T
    W_new = decoupled_update(W, O, hyper.lr, hyper.weight_decay, scale)
    return W_new, M_new, O


def muon_step_batched(Ws, Ms, Gs, hyper: MuonHyper, coeffs, scales,
                      emulate_bf16: bool = False):
    """The batched step: every matrix independently, same hyper-parameters
    and coefficient table (PR #1584 section "Summary": one fused step over all
    matrix parameters).  Returns lists (W', M', O)."""
    outs = [muon_step(W, M, G, hyper, coeffs, s, emulate_bf16)
            for W, M, G, s in zip(Ws, Ms, Gs, scales)]
    return [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs]


def ema_update(E: np.ndarray, P: np.ndarray, decay: float) -> np.ndarray:
    """Step 9: exponential moving average of a parameter tensor,
    E' = d*E + (1-d)*P.

    Pages: PR #1893 table "Architecture and training stack", row "EMA"
    (EMA_DECAY=0.9965); PR #1584 section "Summary" (batched EMA)."""
    E = np.asarray(E, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    return decay * E + (1.0 - decay) * P


def ema_update_batched(Es, Ps, decay: float):
    """EMA over every parameter tensor of the model."""
    return [ema_update(E, P, decay) for E, P in zip(Es, Ps)]


def linear_ramp(v0: float, v1: float, t0: int, t1: int, t: int) -> float:
    """A hyper-parameter that moves linearly from v0 at step t0 to v1 at step
    t1 and holds its end values outside [t0, t1] (t1 <= t0: v0 before t1,
    v1 from t1 on).

    Pages: PR #1893 table "Architecture and training stack", row "Optimizer":
    Muon momentum 0.99 "warmup from 0.92 over 1500 steps".  The page gives the
    end points and the length, not the shape; the straight line between them
    is taken, with step t (0-based, the number of steps already taken) using
    the value at t, so the first step uses 0.92 and step 1500 on uses 0.99.
    """
    if t1 <= t0:
        return float(v1 if t >= t1 else v0)
    f = min(max((t - t0) / (t1 - t0), 0.0), 1.0)
    return float(v0 + (v1 - v0) * f)


def scheduled_hyper(hyper: MuonHyper, mu_ramp, lr_ramp, t: int) -> MuonHyper:
    """The Muon hyper-parameters of step t when momentum and learning rate
    follow ramps (each a (v0, v1, t0, t1) tuple, see linear_ramp)."""
    from dataclasses import replace
    return replace(hyper, momentum=linear_ramp(*mu_ramp, t),
                   lr=linear_ramp(*lr_ramp, t))


@dataclass(frozen=True)
class AdamWHyper:
    """AdamW settings for the non-matrix parameters (embeddings, vectors,
    scalars).  The pages name the optimizer (PR #1893 table "Architecture and
    training stack", row "Optimizer": "AdamW on embeddings/scalars") but give
    none of its settings; these are inputs (the defaults are the commonly
    published AdamW defaults, not values from the pages)."""

    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01


def adamw_update(P, G, M, V, h: AdamWHyper, t: int):
    """One AdamW step (Loshchilov & Hutter's decoupled weight decay with
    Adam's bias-corrected moments), t = 1 for the first step:

      M' = b1 M + (1 - b1) G
      V' = b2 V + (1 - b2) G^2
      P' = P (1 - lr wd) - lr (M' / (1 - b1^t)) / (sqrt(V' / (1 - b2^t)) + eps)

    Returns (P', M', V') in fp64."""
    P = np.asarray(P, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    M_new = h.beta1 * M + (1.0 - h.beta1) * G
    V_new = h.beta2 * V + (1.0 - h.beta2) * G * G
    m_hat = M_new / (1.0 - h.beta1 ** t)
    v_hat = V_new / (1.0 - h.beta2 ** t)
    P_new = P * (1.0 - h.lr * h.weight_decay) - h.lr * m_hat / (np.sqrt(v_hat) + h.eps)
    return P_new, M_new, V_new


def adamw_ema(P, G, M, V, E, h: AdamWHyper, t: int, decay: float):
    """The AdamW step of a non-matrix tensor followed by the EMA of its
    updated value (one pass over the tensor on the GPU side).  The EMA
    follows the optimizer step, so it averages the new parameters (PR #1584
    section "Summary": batched EMA over all parameters after the step).
    Returns (P', M', V', E')."""
    P_new, M_new, V_new = adamw_update(P, G, M, V, h, t)
    return P_new, M_new, V_new, ema_update(E, P_new, decay)


def ns_flops(rows: int, cols: int, steps: int) -> int:
    """Dense Newton-Schulz FLOPs for one matrix: per step 2m^2 n (X X^T) +
    2m^3 (A A) + 2m^2 n (B X) with m = min, n = max."""
    m, n = min(rows, cols), max(rows, cols)
    return steps * (4 * m * m * n + 2 * m * m * m)
