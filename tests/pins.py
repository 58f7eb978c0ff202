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


ALL_PINS = [
    pin_momentum_closed_form, pin_eq_r_row_norms, pin_frobenius,
    pin_ns_diagonal, pin_ns_conjugated, pin_ns_row_vector, pin_ns_band,
    pin_ns_polar_factor, pin_ns_equivariance, pin_update_zero_grad,
    pin_end_to_end_diagonal, pin_step_row_norms, pin_ema_closed_form,
    pin_exact_tiny,
]
