"""Plants plausible mistakes in copies of the oracle (on the CPU) and checks
that each one fails at least one pin, so that the pins can tell a right
oracle from a wrong one."""
import numpy as np
import pytest

import oracle.muon_oracle as mo
import pins


def _ns_drop_c(X, coeffs, round_fn=None):
    X = np.asarray(X, float)
    for a, b, c in coeffs:
        A = X @ X.T
        X = a * X + (b * A) @ X
    return X


def _ns_gram_wrong_side(X, coeffs, round_fn=None):
    # X^T X where X X^T belongs (a shape error unless X is square)
    X = np.asarray(X, float)
    for a, b, c in coeffs:
        A = X.T @ X
        B = b * A + c * A @ A
        X = a * X + B @ X
    return X


def _ns_right_multiply(X, coeffs, round_fn=None):
    # X B where B X belongs (a shape error unless X is square)
    X = np.asarray(X, float)
    for a, b, c in coeffs:
        A = X @ X.T
        B = b * A + c * A @ A
        X = a * X + X @ B
    return X


def _ns_swap_bc(X, coeffs, round_fn=None):
    return mo.__dict__["_orig_ns"](X, [(a, c, b) for a, b, c in coeffs])


def _ns_minus(X, coeffs, round_fn=None):
    X = np.asarray(X, float)
    for a, b, c in coeffs:
        A = X @ X.T
        B = b * A + c * A @ A
        X = a * X - B @ X
    return X


def _ns_one_step_short(X, coeffs, round_fn=None):
    return mo.__dict__["_orig_ns"](X, list(coeffs)[:-1])


def _nesterov_plain(M, G, mu, nesterov=True):
    Mn = mu * np.asarray(M, float) + np.asarray(G, float)
    return Mn, Mn.copy()


def _momentum_lerp(M, G, mu, nesterov=True):
    Mn = mu * np.asarray(M, float) + (1 - mu) * np.asarray(G, float)
    return Mn, np.asarray(G, float) + mu * Mn


def _eq_r_columns(U, eps):
    U = np.asarray(U, float)
    r = np.sqrt(np.sum(U * U, axis=0))
    return U / (r + eps)[None, :]


def _eq_r_eps_in_sqrt(U, eps):
    U = np.asarray(U, float)
    r = np.sqrt(np.sum(U * U, axis=1) + eps)
    return U / r[:, None]


def _frob_squared(X, eps):
    X = np.asarray(X, float)
    return X / (np.sum(X * X) + eps)


def _frob_eps_in_sqrt(X, eps):
    X = np.asarray(X, float)
    return X / np.sqrt(np.sum(X * X) + eps)


def _update_plus(W, O, lr, wd, scale):
    return np.asarray(W, float) * (1 - lr * wd) + lr * scale * np.asarray(O)


def _update_decay_after(W, O, lr, wd, scale):
    return (np.asarray(W, float) - lr * scale * np.asarray(O)) * (1 - lr * wd)


def _update_no_scale(W, O, lr, wd, scale):
    return np.asarray(W, float) * (1 - lr * wd) - lr * np.asarray(O)


def _ema_swapped(E, P, d):
    return (1 - d) * np.asarray(E, float) + d * np.asarray(P, float)


def _step_no_back_transpose(W, M, G, hyper, coeffs, scale,
                            emulate_bf16=False):
    M_new, U = mo.nesterov_momentum(M, G, hyper.momentum, hyper.nesterov)
    if hyper.eq_r:
        U = mo.muon_eq_r(U, hyper.eps_row)
    X, transposed = mo.orient(U)
    X = mo.frobenius_normalize(X, hyper.eps_frob)
    O = mo.newton_schulz(X, coeffs)
    if transposed:
        O = O.T.T.reshape(W.shape)   # forgets to transpose back
    return mo.decoupled_update(W, O, hyper.lr, hyper.weight_decay, scale), \
        M_new, O


def _step_eq_r_after_transpose(W, M, G, hyper, coeffs, scale,
                               emulate_bf16=False):
    M_new, U = mo.nesterov_momentum(M, G, hyper.momentum, hyper.nesterov)
    X, transposed = mo.orient(U)
    if hyper.eq_r:
        X = mo.muon_eq_r(X, hyper.eps_row)
    X = mo.frobenius_normalize(X, hyper.eps_frob)
    O = mo.newton_schulz(X, coeffs)
    if transposed:
        O = O.T
    return mo.decoupled_update(W, O, hyper.lr, hyper.weight_decay, scale), \
        M_new, O


def _ramp_off_by_one(v0, v1, t0, t1, t):
    return mo.__dict__["_orig_ramp"](v0, v1, t0, t1, t + 1)


def _ramp_unclamped(v0, v1, t0, t1, t):
    if t1 <= t0:
        return float(v1 if t >= t1 else v0)
    return float(v0 + (v1 - v0) * (t - t0) / (t1 - t0))


def _adamw_no_bias_correction(P, G, M, V, h, t):
    M2 = h.beta1 * np.asarray(M, float) + (1 - h.beta1) * np.asarray(G, float)
    V2 = h.beta2 * np.asarray(V, float) + (1 - h.beta2) * np.asarray(G, float) ** 2
    return (np.asarray(P, float) * (1 - h.lr * h.weight_decay)
            - h.lr * M2 / (np.sqrt(V2) + h.eps), M2, V2)


def _adamw_l2(P, G, M, V, h, t):
    # weight decay folded into the gradient (Adam + L2) instead of decoupled
    G = np.asarray(G, float) + h.weight_decay * np.asarray(P, float)
    M2 = h.beta1 * np.asarray(M, float) + (1 - h.beta1) * G
    V2 = h.beta2 * np.asarray(V, float) + (1 - h.beta2) * G * G
    mh, vh = M2 / (1 - h.beta1 ** t), V2 / (1 - h.beta2 ** t)
    return np.asarray(P, float) - h.lr * mh / (np.sqrt(vh) + h.eps), M2, V2


def _adamw_swapped_betas(P, G, M, V, h, t):
    from dataclasses import replace
    return mo.__dict__["_orig_adamw"](P, G, M, V,
                                      replace(h, beta1=h.beta2, beta2=h.beta1), t)


def _adamw_step_zero_based(P, G, M, V, h, t):
    return mo.__dict__["_orig_adamw"](P, G, M, V, h, t + 1)


def _adamw_abs_second_moment(P, G, M, V, h, t):
    G = np.asarray(G, float)
    M2 = h.beta1 * np.asarray(M, float) + (1 - h.beta1) * G
    V2 = h.beta2 * np.asarray(V, float) + (1 - h.beta2) * np.abs(G)
    mh, vh = M2 / (1 - h.beta1 ** t), V2 / (1 - h.beta2 ** t)
    return (np.asarray(P, float) * (1 - h.lr * h.weight_decay)
            - h.lr * mh / (np.sqrt(vh) + h.eps), M2, V2)


def _adamw_ema_old_params(P, G, M, V, E, h, t, decay):
    P2, M2, V2 = mo.adamw_update(P, G, M, V, h, t)
    return P2, M2, V2, mo.ema_update(E, P, decay)


MUTANTS = {
    "ns_drop_c": ("newton_schulz", _ns_drop_c),
    "ns_gram_wrong_side": ("newton_schulz", _ns_gram_wrong_side),
    "ns_right_multiply": ("newton_schulz", _ns_right_multiply),
    "ns_swap_bc": ("newton_schulz", _ns_swap_bc),
    "ns_minus": ("newton_schulz", _ns_minus),
    "ns_one_step_short": ("newton_schulz", _ns_one_step_short),
    "nesterov_plain": ("nesterov_momentum", _nesterov_plain),
    "momentum_lerp": ("nesterov_momentum", _momentum_lerp),
    "eq_r_columns": ("muon_eq_r", _eq_r_columns),
    "eq_r_eps_in_sqrt": ("muon_eq_r", _eq_r_eps_in_sqrt),
    "frob_squared": ("frobenius_normalize", _frob_squared),
    "frob_eps_in_sqrt": ("frobenius_normalize", _frob_eps_in_sqrt),
    "update_plus": ("decoupled_update", _update_plus),
    "update_decay_after": ("decoupled_update", _update_decay_after),
    "update_no_scale": ("decoupled_update", _update_no_scale),
    "ema_swapped": ("ema_update", _ema_swapped),
    "step_no_back_transpose": ("muon_step", _step_no_back_transpose),
    "step_eq_r_after_transpose": ("muon_step", _step_eq_r_after_transpose),
    "ramp_off_by_one": ("linear_ramp", _ramp_off_by_one),
    "ramp_unclamped": ("linear_ramp", _ramp_unclamped),
    "adamw_no_bias_correction": ("adamw_update", _adamw_no_bias_correction),
    "adamw_l2": ("adamw_update", _adamw_l2),
    "adamw_swapped_betas": ("adamw_update", _adamw_swapped_betas),
    "adamw_step_zero_based": ("adamw_update", _adamw_step_zero_based),
    "adamw_abs_second_moment": ("adamw_update", _adamw_abs_second_moment),
    "adamw_ema_old_params": ("adamw_ema", _adamw_ema_old_params),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setitem(mo.__dict__, "_orig_ns", mo.newton_schulz)
    monkeypatch.setitem(mo.__dict__, "_orig_ramp", mo.linear_ramp)
    monkeypatch.setitem(mo.__dict__, "_orig_adamw", mo.adamw_update)
    monkeypatch.setattr(mo, attr, fn)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mo)
        except Exception as e:  # AssertionError or a shape error
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"mutant {name} passed every pin"
