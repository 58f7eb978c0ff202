"""Pins for the fp64 oracle: checks that tie it to something other than
itself (closed forms, invariants, LAPACK SVD, exact rational arithmetic).

Each pin takes the oracle module as an argument so that the mutation test
can run the same pins against deliberately broken copies of the oracle and
show that every planted mistake fails at least one pin.
"""

from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
FIXED = (3.4445, -4.7750, 2.0315)


def _scalar_poly_chain(sig, coeffs):
    """Scalar iteration x <- a x + b x^3 + c x^5 applied elementwise."""
    x = np.array(sig, dtype=np.float64)
    for a, b, c in coeffs:
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def _hyper(o, **kw):
    base = dict(momentum=0.9, lr=0.05, weight_decay=0.1, eps_row=0.0,
                eps_frob=0.0, nesterov=True, eq_r=True)
    base.update(kw)
    return o.MuonHyper(**base)


# ---------------------------------------------------------------- momentum
def pin_momentum_closed_form(o):
    """Constant G, M0 = 0: M_t = G (1 - mu^t) / (1 - mu) and the Nesterov
    look-ahead U_t = G + mu M_t."""
    rng = np.random.default_rng(0)
    G = rng.standard_normal((5, 7))
    mu = 0.9
    M = np.zeros_like(G)
    for t in range(1, 8):
        M, U = o.nesterov_momentum(M, G, mu, True)
        Mt = G * (1 - mu ** t) / (1 - mu)
        assert np.allclose(M, Mt, rtol=1e-13, atol=0)
        assert np.allclose(U, G * (1 + mu * (1 - mu ** t) / (1 - mu)),
                           rtol=1e-13, atol=0)
    # Without Nesterov the update direction is the buffer itself.
    M2, U2 = o.nesterov_momentum(np.zeros_like(G), G, mu, False)
    assert np.array_equal(U2, M2) and np.allclose(M2, G)


# ---------------------------------------------------------------- MuonEq-R
def pin_eq_r_row_norms(o):
    """After MuonEq-R every stored row has norm r/(r+eps); zero rows stay
    zero; the direction of each row is unchanged."""
    rng = np.random.default_rng(1)
    U = rng.standard_normal((6, 9)) * np.exp(rng.standard_normal(6))[:, None]
    U[3] = 0.0
    eps = 1e-3
    X = o.muon_eq_r(U, eps)
    r = np.array([np.sqrt(sum(v * v for v in row)) for row in U])
    got = np.array([np.sqrt(sum(v * v for v in row)) for row in X])
    assert np.allclose(got, r / (r + eps), rtol=1e-13)
    assert np.all(X[3] == 0)
    for i in (0, 1, 2, 4, 5):   # same direction
        assert np.allclose(X[i] * (r[i] + eps), U[i], rtol=1e-12)
    # A non-square case: the norm is over rows, not columns.
    with np.errstate(invalid="ignore"):
        X0 = o.muon_eq_r(U, 0.0)
    keep = [i for i in range(6) if i != 3]
    assert np.allclose(np.linalg.norm(X0[keep], axis=1), 1.0, rtol=1e-13)


# ---------------------------------------------------------------- Frobenius
def pin_frobenius(o):
    rng = np.random.default_rng(2)
    X = rng.standard_normal((4, 11)) * 37.0
    for eps in (0.0, 1e-7, 0.5):
        Y = o.frobenius_normalize(X, eps)
        f = np.sqrt(np.sum(X ** 2))
        assert abs(np.sqrt(np.sum(Y ** 2)) - f / (f + eps)) < 1e-13
        assert np.allclose(Y * (f + eps), X, rtol=1e-12)


# ---------------------------------------------------------------- NS
def pin_ns_diagonal(o):
    """X = [diag(s) 0] (m x n): Newton-Schulz acts on each singular value
    by the scalar polynomial chain."""
    sig = np.array([1.0, 0.7, 0.31, 0.05, 1e-3])
    m, n = 5, 9
    X = np.zeros((m, n))
    X[np.arange(m), np.arange(m)] = sig
    for coeffs in ([FIXED] * 5, [(1.875, -1.25, 0.375)] * 3,
                   [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5)]):
        Y = o.newton_schulz(X, coeffs)
        want = np.zeros((m, n))
        want[np.arange(m), np.arange(m)] = _scalar_poly_chain(sig, coeffs)
        assert np.allclose(Y, want, rtol=1e-12, atol=1e-14)


def pin_ns_conjugated(o):
    """X = Q [diag(s) 0] V^T with random orthogonal Q, V gives
    Q [diag(p(s)) 0] V^T: Newton-Schulz commutes with orthogonal
    conjugation and acts on singular values only."""
    rng = np.random.default_rng(3)
    m, n = 6, 10
    Q, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, n)))
    sig = np.array([0.9, 0.6, 0.4, 0.2, 0.1, 0.02])
    S = np.zeros((m, n))
    S[np.arange(m), np.arange(m)] = sig
    X = Q @ S @ V.T
    coeffs = [FIXED] * 5
    P = np.zeros((m, n))
    P[np.arange(m), np.arange(m)] = _scalar_poly_chain(sig, coeffs)
    Y = o.newton_schulz(X, coeffs)
    assert np.allclose(Y, Q @ P @ V.T, rtol=0, atol=1e-12)


def pin_ns_row_vector(o):
    """1 x n input of unit norm: its one singular value is 1, so the output
    is the scalar chain evaluated at 1 times the input (for one step that is
    a + b + c)."""
    rng = np.random.default_rng(4)
    g = rng.standard_normal((1, 13))
    X = g / np.linalg.norm(g)
    coeffs = [FIXED, (1.875, -1.25, 0.375), (2.0, -0.5, 0.25)]
    Y = o.newton_schulz(X, coeffs)
    f = _scalar_poly_chain([1.0], coeffs)[0]
    assert np.allclose(Y, f * X, rtol=1e-13)
    a, b, c = FIXED
    assert np.allclose(o.newton_schulz(X, [FIXED]), (a + b + c) * X,
                       rtol=1e-13)


def pin_ns_band(o):
    """Singular values of the output (LAPACK SVD) lie inside the range of the
    composed scalar polynomial over [sigma_min(X), 1]."""
    rng = np.random.default_rng(5)
    for m, n in ((16, 40), (24, 24)):
        X = rng.standard_normal((m, n))
        X /= np.linalg.norm(X)
        s_in = np.linalg.svd(X, compute_uv=False)
        coeffs = [FIXED] * 5
        s_out = np.linalg.svd(o.newton_schulz(X, coeffs), compute_uv=False)
        grid = np.linspace(s_in.min(), 1.0, 200001)
        p = _scalar_poly_chain(grid, coeffs)
        assert s_out.min() >= p.min() - 1e-9
        assert s_out.max() <= p.max() + 1e-9
        # and exactly the chain applied to each input singular value
        assert np.allclose(np.sort(s_out),
                           np.sort(np.abs(_scalar_poly_chain(s_in, coeffs))),
                           rtol=1e-9)


def pin_ns_polar_factor(o):
    """The classical quintic (15/8, -10/8, 3/8) iterated on a well-conditioned
    input converges to the polar factor U V^T from the SVD."""
    rng = np.random.default_rng(6)
    m, n = 8, 20
    Q, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, n)))
    S = np.zeros((m, n))
    S[np.arange(m), np.arange(m)] = np.linspace(0.3, 1.0, m)
    X = Q @ S @ V.T
    Y = o.newton_schulz(X, [(15 / 8, -10 / 8, 3 / 8)] * 40)
    Uu, _, Vt = np.linalg.svd(X, full_matrices=False)
    assert np.allclose(Y, Uu @ Vt, atol=1e-12)


def pin_polar_express_table(o_pe):
    """The generated Polar-Express-style table: each step equioscillates on
    its design interval (4 alternation points: the minimax certificate), each
    nominal interval is the image of the previous one, and the composed
    schedule maps [lo0, 1] into the last image."""
    with open(os.path.join(HERE, "golden", "polar_express_k4.json")) as f:
        doc = json.load(f)
    rows, intervals = doc["coeffs"], doc["intervals"]
    design = doc["design_intervals"]
    assert len(rows) == 4
    for (a, b, c), (lo, hi) in zip(rows, design):
        x = np.linspace(lo, hi, 400001)
        e = 1.0 - (a * x + b * x ** 3 + c * x ** 5)
        E = np.max(np.abs(e))
        near = np.abs(np.abs(e) - E) < 1e-9 * max(1.0, E)
        signs = np.sign(e[np.flatnonzero(near)])
        alternations = 1 + int(np.sum(signs[1:] != signs[:-1]))
        assert alternations >= 4, (alternations, lo, hi)
        assert abs(e[0] - E) < 1e-9 and abs(e[-1] + E) < 1e-9
    for k in range(3):
        a, b, c = rows[k]
        lo, hi = intervals[k]
        x = np.linspace(lo, hi, 400001)
        y = a * x + b * x ** 3 + c * x ** 5
        assert abs(y.min() - intervals[k + 1][0]) < 1e-8
        assert abs(y.max() - intervals[k + 1][1]) < 1e-8
    rows2, iv2, d2 = o_pe.polar_express_table(
        4, *doc["initial_interval"], doc["cushion"], doc["inflate"])
    assert np.allclose(np.array(rows2), np.array(rows), rtol=1e-12)
    assert np.allclose(np.array(iv2), np.array(intervals), rtol=1e-12)
    assert np.allclose(np.array(d2), np.array(design), rtol=1e-12)
    lo0, hi0 = doc["initial_interval"]
    x = np.geomspace(lo0, hi0, 20001)
    y = _scalar_poly_chain(x, rows)
    a, b, c = rows[-1]
    lo3, hi3 = intervals[-1]
    g = np.linspace(lo3, hi3, 400001)
    p = a * g + b * g ** 3 + c * g ** 5
    assert y.min() >= p.min() - 1e-9 and y.max() <= p.max() + 1e-9
    # the recorded composed band is the range of the scalar chain over the
    # initial interval (dense sampling, geometric and linear, from below)
    xs = np.concatenate([np.geomspace(lo0, hi0, 400001), np.linspace(lo0, hi0, 400001)])
    ys = _scalar_poly_chain(xs, rows)
    band = doc["band"]
    assert band[0] <= ys.min() + 1e-12 and ys.max() <= band[1] + 1e-12
    assert ys.min() - band[0] < 1e-6 and band[1] - ys.max() < 1e-6
    # the design interval tracks the true lower end: four different steps
    for i in range(4):
        for j in range(i + 1, 4):
            assert np.max(np.abs(np.array(rows[i]) - np.array(rows[j]))) > 1e-3
    # the plain greedy chain (no margins) equioscillates around 1 on the
    # whole initial interval: its band is [1 - E, 1 + E], narrower than the
    # table's margin-widened band
    plain, _, _ = o_pe.polar_express_table(4, lo0, hi0)
    yp = _scalar_poly_chain(xs, plain)
    pb = doc["band_plain_greedy"]
    assert abs(yp.min() - pb[0]) < 1e-6 and abs(yp.max() - pb[1]) < 1e-6
    assert abs((pb[0] + pb[1]) - 2.0) < 1e-9
    assert pb[0] >= band[0] and pb[1] <= band[1]
    # the plain greedy schedule (no margins) is a minimax chain too
    r0, iv0, _ = o_pe.polar_express_table(2, 1e-3, 1.0)
    (a, b, c) = r0[0]
    assert abs((a * 1e-3 + b * 1e-9 + c * 1e-15) - iv0[1][0]) < 1e-12


def pin_ns_equivariance(o):
    """With MuonEq-R off: O(G^T) = O(G)^T, and O(alpha G) = O(G) for
    alpha > 0 from zero momentum (eps = 0)."""
    rng = np.random.default_rng(7)
    h = _hyper(o, eq_r=False, weight_decay=0.0)
    for r, c in ((6, 10), (10, 6), (7, 7)):
        G = rng.standard_normal((r, c))
        W = np.zeros((r, c))
        _, _, O1 = o.muon_step(W, np.zeros((r, c)), G, h, [FIXED] * 3, 1.0)
        _, _, O2 = o.muon_step(W.T, np.zeros((c, r)), G.T, h, [FIXED] * 3,
                               1.0)
        assert np.allclose(O2, O1.T, atol=1e-12)
        _, _, O3 = o.muon_step(W, np.zeros((r, c)), 3.7 * G, h, [FIXED] * 3,
                               1.0)
        assert np.allclose(O3, O1, atol=1e-12)


# ---------------------------------------------------------------- update
def pin_update_zero_grad(o):
    """G = 0 and M = 0: the update direction is zero and only the decoupled
    decay acts, W_t = W_0 (1 - lr wd)^t."""
    rng = np.random.default_rng(8)
    W0 = rng.standard_normal((5, 8))
    h = _hyper(o, eps_row=1e-7, eps_frob=1e-7)
    W, M = W0.copy(), np.zeros_like(W0)
    for t in range(1, 5):
        W, M, O = o.muon_step(W, M, np.zeros_like(W0), h, [FIXED] * 5, 2.0)
        assert np.all(O == 0) and np.all(M == 0)
        assert np.allclose(W, W0 * (1 - h.lr * h.weight_decay) ** t,
                           rtol=1e-14)


def pin_end_to_end_diagonal(o):
    """Whole step on a diagonal gradient.  G = diag(g), g > 0, M = 0:
    U = (1 + mu) G, MuonEq-R gives the identity, the Frobenius step gives
    I/sqrt(m), Newton-Schulz gives p(1/sqrt(m)) I, and
    W' = W (1 - lr wd) - lr scale p(1/sqrt(m)) I."""
    rng = np.random.default_rng(9)
    for m, W_shape in ((6, (6, 6)),):
        g = rng.uniform(0.5, 2.0, m)
        G = np.diag(g)
        W = rng.standard_normal(W_shape)
        h = _hyper(o)
        coeffs = [FIXED] * 5
        W1, M1, O = o.muon_step(W, np.zeros(W_shape), G, h, coeffs, 1.7)
        p = _scalar_poly_chain([1 / np.sqrt(m)], coeffs)[0]
        assert np.allclose(O, p * np.eye(m), atol=1e-12)
        assert np.allclose(M1, G)
        want = W * (1 - h.lr * h.weight_decay) - h.lr * 1.7 * p * np.eye(m)
        assert np.allclose(W1, want, atol=1e-12)
    # Rectangular, transposed orientation: G = [diag(g); 0] (rows > cols).
    g = rng.uniform(0.5, 2.0, 4)
    G = np.zeros((7, 4))
    G[np.arange(4), np.arange(4)] = g
    W = rng.standard_normal((7, 4))
    h = _hyper(o, eps_row=1e-30)
    W1, _, O = o.muon_step(W, np.zeros((7, 4)), G, h, [FIXED] * 5, 1.0)
    # zero rows stay zero; the 4 unit rows give X = I_4-padded / 2
    p = _scalar_poly_chain([0.5], [FIXED] * 5)[0]
    want_O = np.zeros((7, 4))
    want_O[np.arange(4), np.arange(4)] = p
    assert np.allclose(O, want_O, atol=1e-12)


def pin_step_row_norms(o):
    """With no Newton-Schulz step the update is the normalised look-ahead
    itself, so with MuonEq-R on every stored row of O has the same norm
    1/sqrt(rows), in both orientations."""
    rng = np.random.default_rng(12)
    h = _hyper(o, eps_row=0.0, eps_frob=0.0)
    for r, c in ((9, 4), (4, 9), (5, 5)):
        G = rng.standard_normal((r, c)) * np.exp(rng.standard_normal(r))[:, None]
        _, _, O = o.muon_step(np.zeros((r, c)), np.zeros((r, c)), G, h, [],
                              1.0)
        assert O.shape == (r, c)
        assert np.allclose(np.linalg.norm(O, axis=1), 1 / np.sqrt(r),
                           rtol=1e-12)


def pin_ema_closed_form(o):
    """Constant P: E_t = P + d^t (E_0 - P)."""
    rng = np.random.default_rng(10)
    P = rng.standard_normal(17)
    E0 = rng.standard_normal(17)
    d = 0.9965
    E = E0.copy()
    for t in range(1, 40):
        E = o.ema_update(E, P, d)
        assert np.allclose(E, P + d ** t * (E0 - P), rtol=1e-12, atol=1e-15)
    Es = o.ema_update_batched([E0, 2 * E0], [P, P], 0.5)
    assert np.allclose(Es[1], P + 0.5 * (2 * E0 - P))


# ---------------------------------------------------------------- exact
def _fmat(a):
    return [[Fraction(v) for v in row] for row in a]


def _mm(A, B):
    n, k, m = len(A), len(B), len(B[0])
    return [[sum(A[i][t] * B[t][j] for t in range(k)) for j in range(m)]
            for i in range(n)]


def _tr(A):
    return [list(r) for r in zip(*A)]


def _exact_step(W, M, G, mu, lr, wd, scale, coeffs, eq_r):
    """Whole step in exact rational arithmetic with hand-written loops
    (inputs chosen so that every norm is rational; eps = 0)."""
    rows, cols = len(G), len(G[0])
    Mn = [[mu * M[i][j] + G[i][j] for j in range(cols)] for i in range(rows)]
    U = [[G[i][j] + mu * Mn[i][j] for j in range(cols)] for i in range(rows)]

    def ratsqrt(q):
        num, den = q.numerator, q.denominator
        rn, rd = int(round(num ** 0.5)), int(round(den ** 0.5))
        assert rn * rn == num and rd * rd == den, "norm not rational"
        return Fraction(rn, rd)

    if eq_r:
        for i in range(rows):
            r = ratsqrt(sum(v * v for v in U[i]))
            if r != 0:
                U[i] = [v / r for v in U[i]]
    X = _tr(U) if rows > cols else [list(r) for r in U]
    f = ratsqrt(sum(v * v for row in X for v in row))
    X = [[v / f for v in row] for row in X]
    for a, b, c in coeffs:
        A = _mm(X, _tr(X))
        AA = _mm(A, A)
        B = [[b * A[i][j] + c * AA[i][j] for j in range(len(A))]
             for i in range(len(A))]
        BX = _mm(B, X)
        X = [[a * X[i][j] + BX[i][j] for j in range(len(X[0]))]
             for i in range(len(X))]
    O = _tr(X) if rows > cols else X
    Wn = [[W[i][j] * (1 - lr * wd) - lr * scale * O[i][j]
           for j in range(cols)] for i in range(rows)]
    return Wn, Mn, O


def pin_exact_tiny(o):
    """Brute force on tiny inputs: exact rationals vs the fp64 oracle."""
    coeffs = [(Fraction("3.4445"), Fraction("-4.7750"), Fraction("2.0315")),
              (Fraction(15, 8), Fraction(-10, 8), Fraction(3, 8))]
    fcoeffs = [tuple(float(v) for v in r) for r in coeffs]
    mu, lr, wd, scale = Fraction(1, 2), Fraction(1, 20), Fraction(1, 10), \
        Fraction(3, 2)
    cases = [
        # 4 x 5, MuonEq-R on: integer row norms 3, 7, 9, 11 (x 3/2 from the
        # Nesterov factor); four unit rows give ||X||_F = 2.
        ([[1, 2, 2, 0, 0], [2, 3, 0, 6, 0], [0, 1, 4, 0, 8],
          [6, 0, 2, 0, 9]], True),
        # 5 x 4 (transposed orientation), MuonEq-R off; ||G||_F = 13.
        ([[3, 4, 0, 0], [0, 0, 12, 0], [0, 0, 0, 0], [0, 0, 0, 0],
          [0, 0, 0, 0]], False),
        # 9 x 4 (transposed orientation), MuonEq-R on: nine integer row
        # norms, so ||X||_F = 3.
        ([[1, 2, 2, 0], [2, 3, 6, 0], [0, 1, 4, 8], [6, 0, 2, 9],
          [4, 4, 7, 0], [0, 2, 6, 9], [2, 10, 11, 0], [1, 0, 2, 2],
          [3, 0, 0, 4]], True),
        # 1 x 6 row vector, MuonEq-R on.
        ([[2, -3, 6, 0, 0, 0]], True),
        # 2 x 3, MuonEq-R off; ||G||_F = 5.
        ([[1, 2, 2], [4, 0, 0]], False),
    ]
    rng = np.random.default_rng(11)
    for Gi, eq_r in cases:
        rows, cols = len(Gi), len(Gi[0])
        G = _fmat(Gi)
        M = [[Fraction(0)] * cols for _ in range(rows)]
        W = [[Fraction(int(v), 64) for v in row]
             for row in rng.integers(-9, 10, (rows, cols))]
        Wn, Mn, O = _exact_step(W, M, G, mu, lr, wd, scale, coeffs, eq_r)
        h = o.MuonHyper(momentum=0.5, lr=0.05, weight_decay=0.1, eps_row=0.0,
                        eps_frob=0.0, nesterov=True, eq_r=eq_r)
        fW = np.array([[float(v) for v in r] for r in W])
        fG = np.array([[float(v) for v in r] for r in G])
        W1, M1, O1 = o.muon_step(fW, np.zeros_like(fG), fG, h, fcoeffs, 1.5)
        assert np.allclose(O1, np.array(O, dtype=float), rtol=1e-12,
                           atol=1e-13)
        assert np.allclose(W1, np.array(Wn, dtype=float), rtol=1e-12,
                           atol=1e-13)
        assert np.allclose(M1, np.array(Mn, dtype=float), rtol=1e-14)


# ---------------------------------------------------------------- schedules
def pin_ramp(o):
    """Linear ramp: end values at and beyond the ends, the mean at the
    midpoint, equal increments per step inside, a step function when the
    ramp has no length; the pages' momentum warm-up (0.92 -> 0.99 over 1500
    steps) at its first, middle and last steps."""
    r = o.linear_ramp
    assert r(0.92, 0.99, 0, 1500, 0) == 0.92
    assert abs(r(0.92, 0.99, 0, 1500, 750) - 0.955) < 1e-15
    assert r(0.92, 0.99, 0, 1500, 1500) == 0.99
    assert r(0.92, 0.99, 0, 1500, 10 ** 6) == 0.99
    assert r(0.5, 1.5, 10, 20, 3) == 0.5          # before the start
    vals = [r(0.5, 1.5, 10, 20, t) for t in range(10, 21)]
    assert np.allclose(np.diff(vals), 0.1, rtol=0, atol=1e-15)
    assert r(2.0, 3.0, 5, 5, 4) == 2.0 and r(2.0, 3.0, 5, 5, 5) == 3.0
    h = o.scheduled_hyper(o.MuonHyper(momentum=0.5, lr=9.0),
                          (0.92, 0.99, 0, 1500), (0.02, 0.01, 100, 200), 150)
    assert abs(h.momentum - (0.92 + 0.07 * 0.1)) < 1e-15
    assert abs(h.lr - 0.015) < 1e-15


def pin_ramp_momentum_exact(o):
    """Momentum under a ramped mu, checked in exact rational arithmetic:
    with constant G and M_0 = 0, M_T = G * sum_s prod_{k=s+1..T} mu_k where
    step k (1-based) uses mu at ramp step k - 1."""
    v0, v1, t0, t1 = Fraction(1, 2), Fraction(7, 8), 0, 3
    def mu_exact(t):
        if t >= t1:
            return v1
        return v0 + (v1 - v0) * Fraction(t - t0, t1 - t0)
    G = Fraction(3, 1)
    T = 5
    expect = sum(G * np.prod([mu_exact(k - 1) for k in range(s + 1, T + 1)] or [1])
                 for s in range(1, T + 1))
    M = np.zeros(1)
    for t in range(T):
        mu = o.linear_ramp(float(v0), float(v1), t0, t1, t)
        assert abs(mu - float(mu_exact(t))) < 1e-15
        M, _ = o.nesterov_momentum(M, np.array([float(G)]), mu, True)
    assert abs(M[0] - float(expect)) < 1e-12


# ---------------------------------------------------------------- AdamW
def _adamw_h(o, **kw):
    base = dict(lr=0.01, beta1=0.9, beta2=0.99, eps=0.0, weight_decay=0.1)
    base.update(kw)
    return o.AdamWHyper(**base)


def pin_adamw_first_and_constant_steps(o):
    """From zero moments with eps = 0 the bias-corrected moments of a
    constant gradient are g and g^2 at every step, so each step moves every
    entry by lr * sign(g) after the decoupled decay:
    P_T = P_0 c^T - lr sign(g) (1 + c + ... + c^(T-1)),  c = 1 - lr wd."""
    rng = np.random.default_rng(20)
    P0 = rng.standard_normal(9)
    g = rng.standard_normal(9)
    h = _adamw_h(o)
    c = 1 - h.lr * h.weight_decay
    P, M, V = P0.copy(), np.zeros(9), np.zeros(9)
    for T in range(1, 12):
        P, M, V = o.adamw_update(P, g, M, V, h, T)
        geo = sum(c ** k for k in range(T))
        assert np.allclose(P, P0 * c ** T - h.lr * np.sign(g) * geo,
                           rtol=1e-12, atol=1e-14)
        assert np.allclose(M, g * (1 - h.beta1 ** T), rtol=1e-12)
        assert np.allclose(V, g * g * (1 - h.beta2 ** T), rtol=1e-12)


def pin_adamw_exact_two_steps(o):
    """Two AdamW steps in exact rational arithmetic with b1 = 1/2, b2 = 1/2
    and gradients (5, 1): the bias-corrected second moment of step 2 is
    (b2 g1^2 + g2^2) / (1 + b2) = 9, a perfect square, so the whole update is
    rational."""
    F = Fraction
    b1, b2, lr, wd = F(1, 2), F(1, 2), F(1, 10), F(1, 5)
    g1, g2, p0 = F(5), F(1), F(3)
    m1 = (1 - b1) * g1
    v1 = (1 - b2) * g1 * g1
    p1 = p0 * (1 - lr * wd) - lr * (m1 / (1 - b1)) / F(5)     # sqrt(v1/(1-b2)) = 5
    m2 = b1 * m1 + (1 - b1) * g2
    v2 = b2 * v1 + (1 - b2) * g2 * g2
    assert v2 / (1 - b2 ** 2) == 9
    p2 = p1 * (1 - lr * wd) - lr * (m2 / (1 - b1 ** 2)) / F(3)
    h = o.AdamWHyper(lr=0.1, beta1=0.5, beta2=0.5, eps=0.0, weight_decay=0.2)
    P, M, V = o.adamw_update(np.array([3.0]), np.array([5.0]), np.zeros(1),
                             np.zeros(1), h, 1)
    assert abs(P[0] - float(p1)) < 1e-15
    P, M, V = o.adamw_update(P, np.array([1.0]), M, V, h, 2)
    assert abs(P[0] - float(p2)) < 1e-15 and abs(M[0] - float(m2)) < 1e-15
    assert abs(V[0] - float(v2)) < 1e-15


def pin_adamw_invariances(o):
    """With eps = 0 the AdamW direction is unchanged by a positive rescaling
    of every gradient and flips with their sign; with lr = 0 nothing moves
    but the moments."""
    rng = np.random.default_rng(21)
    P = rng.standard_normal(6)
    G1, G2 = rng.standard_normal(6), rng.standard_normal(6)
    h = _adamw_h(o)
    def run(s):
        p, m, v = P.copy(), np.zeros(6), np.zeros(6)
        p, m, v = o.adamw_update(p, s * G1, m, v, h, 1)
        p, m, v = o.adamw_update(p, s * G2, m, v, h, 2)
        return p
    base = run(1.0)
    assert np.allclose(run(37.5), base, rtol=1e-12)
    c2 = (1 - h.lr * h.weight_decay) ** 2
    assert np.allclose(run(-1.0) - P * c2, -(base - P * c2), rtol=1e-12)
    p, _, _ = o.adamw_update(P, G1, np.zeros(6), np.zeros(6),
                             _adamw_h(o, lr=0.0), 1)
    assert np.array_equal(p, P)


def pin_adamw_ema(o):
    """The fused pass: the EMA averages the updated parameters,
    E' = d E + (1 - d) P' (checked against the AdamW closed form of a first
    step, P' = P c - lr sign(g))."""
    rng = np.random.default_rng(22)
    P, G, E = rng.standard_normal(5), rng.standard_normal(5), rng.standard_normal(5)
    h = _adamw_h(o)
    d = 0.9965
    P1, M1, V1, E1 = o.adamw_ema(P, G, np.zeros(5), np.zeros(5), E, h, 1, d)
    Pc = P * (1 - h.lr * h.weight_decay) - h.lr * np.sign(G)
    assert np.allclose(P1, Pc, rtol=1e-12, atol=1e-15)
    assert np.allclose(E1, d * E + (1 - d) * Pc, rtol=1e-12, atol=1e-15)


ALL_PINS = [
    pin_momentum_closed_form, pin_eq_r_row_norms, pin_frobenius,
    pin_ns_diagonal, pin_ns_conjugated, pin_ns_row_vector, pin_ns_band,
    pin_ns_polar_factor, pin_ns_equivariance, pin_update_zero_grad,
    pin_end_to_end_diagonal, pin_step_row_norms, pin_ema_closed_form,
    pin_exact_tiny, pin_ramp, pin_ramp_momentum_exact,
    pin_adamw_first_and_constant_steps, pin_adamw_exact_two_steps,
    pin_adamw_invariances, pin_adamw_ema,
]
