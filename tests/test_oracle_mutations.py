"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the CPU oracle (in memory, by replacing one of its
functions for the duration of the test) and runs every pin of test_oracle_pins.py: at
least one pin must fail.  A case that no pin catches means a part of the oracle that
nothing outside it fixes.  The clean oracle must pass every pin.

Not planted, because they are not mistakes: the right-Gram form of the NS update
(X (b A' + c A'^2) with A' = X^T X equals (b A + c A^2) X with A = X X^T, since
(X X^T)^k X = X (X^T X)^k), and the choice of side for square matrices.
"""
import inspect

import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import nshb_oracle as o

ORIG = {name: getattr(o, name) for name in (
    "fro", "coeff_table", "momentum", "newton_schulz", "scalar_ns", "msgn_svd", "shape_scale", "muon_apply",
    "hyperball_apply", "radial_brake_apply", "relative_update_apply", "adam_update", "himuon_ns", "ridge_lambda",
    "newton_precondition")}


def pin_cases():
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != pins.__name__:
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            yield name, fn, ()
            continue
        for v in marks[0].args[1]:
            yield name, fn, (v,)


def failing_pins():
    failed = []
    for name, fn, args in pin_cases():
        try:
            with np.errstate(all="ignore"):
                fn(*args)
        except Exception:  # a failed assertion, or an error the mistake provokes
            failed.append(name)
    return failed


def _raw_iteration(X, steps, coeffs):
    for a, b, c in o.coeff_table(steps, coeffs):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X


# ---------------------------------------------------------------- planted mistakes
def nesterov_from_old_buffer(M, G, beta, nesterov=True):
    M_new, U = ORIG["momentum"](M, G, beta, nesterov)
    if nesterov:
        U = (1 - beta) * np.asarray(G, float) + beta * np.asarray(M, float)
    return M_new, U


def plain_momentum_from_old_buffer(M, G, beta, nesterov=True):
    M_new, U = ORIG["momentum"](M, G, beta, nesterov)
    return M_new, (U if nesterov else np.asarray(M, float).copy())


def ns_sign_of_b(G, steps=5, eps=o.NS_EPS, coeffs=None):
    return ORIG["newton_schulz"](G, steps, eps, [(a, -b, c) for a, b, c in o.coeff_table(steps, coeffs)])


def ns_without_c(G, steps=5, eps=o.NS_EPS, coeffs=None):
    return ORIG["newton_schulz"](G, steps, eps, [(a, b, 0.0) for a, b, c in o.coeff_table(steps, coeffs)])


def ns_one_iteration_short(G, steps=5, eps=o.NS_EPS, coeffs=None):
    return ORIG["newton_schulz"](G, steps - 1, eps, o.coeff_table(steps, coeffs)[:-1])


def ns_without_eps(G, steps=5, eps=o.NS_EPS, coeffs=None):
    return ORIG["newton_schulz"](G, steps, 0.0, coeffs)


def ns_spectral_normalisation(G, steps=5, eps=o.NS_EPS, coeffs=None):
    X = np.asarray(G, float)
    tall = X.shape[0] > X.shape[1]
    X = X.T if tall else X
    X = _raw_iteration(X / (np.linalg.norm(X, 2) + eps), steps, coeffs)
    return np.ascontiguousarray(X.T if tall else X)


def coefficient_table_reversed(steps, coeffs=None):
    return ORIG["coeff_table"](steps, coeffs)[::-1]


def scalar_map_sign_of_b(sigma, steps=5, coeffs=None):
    return ORIG["scalar_ns"](sigma, steps, [(a, -b, c) for a, b, c in o.coeff_table(steps, coeffs)])


def msgn_rows_and_columns_reversed(G):
    G = np.asarray(G, float)
    return ORIG["msgn_svd"](G.T).T[::-1, ::-1].copy()


def muon_decay_without_lr(W, O, lr, weight_decay=0.0):
    W = np.asarray(W, float)
    return ORIG["muon_apply"](W, O, lr, 0.0) - weight_decay * W


def brake_target_from_the_new_norm(W, O, lr, outward, inward, eps=o.HB_EPS):
    w_prev = np.asarray(W, float)
    w = ORIG["muon_apply"](w_prev, O, lr, 0.0)
    n_prev, n_new = ORIG["fro"](w_prev), ORIG["fro"](w)
    delta = n_new - n_prev
    s = outward if delta > 0 else inward
    return w * ((n_new + s * delta) / n_new)


def fro_without_sqrt(x):
    return float(np.sum(np.asarray(x, float) ** 2))


def shape_scale_inverted(rows, cols):
    return ORIG["shape_scale"](cols, rows)


def muon_ignores_weight_decay(W, O, lr, weight_decay=0.0):
    return ORIG["muon_apply"](W, O, lr, 0.0)


def hyperball_adds_the_step(W, O, eta, rho, eps=o.HB_EPS):
    return ORIG["hyperball_apply"](W, -np.asarray(O, float), eta, rho, eps)


def hyperball_unnormalised_update(W, O, eta, rho, eps=o.HB_EPS):
    return ORIG["hyperball_apply"](W, O, eta * ORIG["fro"](O), rho, eps)


def hyperball_ignores_radius(W, O, eta, rho, eps=o.HB_EPS):
    return ORIG["hyperball_apply"](W, O, eta, None, eps)


def hyperball_without_reprojection(W, O, eta, rho, eps=o.HB_EPS):
    W = np.asarray(W, float)
    O = np.asarray(O, float)
    return W - eta * O / max(ORIG["fro"](O), eps), False


def brake_factors_swapped(W, O, lr, outward, inward, eps=o.HB_EPS):
    return ORIG["radial_brake_apply"](W, O, lr, inward, outward, eps)


def relative_update_unnormalised(W, O, lr, weight_decay=0.0, eps=o.HB_EPS):
    W = np.asarray(W, float)
    return (1 - lr * weight_decay) * W - lr * ORIG["fro"](W) * np.asarray(O, float)


def adam_without_bias_correction(M, V, G, t, beta1=o.ADAM_BETA1, beta2=o.ADAM_BETA2, eps=o.ADAM_EPS):
    M_new, V_new, _ = ORIG["adam_update"](M, V, G, t, beta1, beta2, eps)
    return M_new, V_new, M_new / (np.sqrt(V_new) + eps)


def adam_second_moment_of_g(M, V, G, t, beta1=o.ADAM_BETA1, beta2=o.ADAM_BETA2, eps=o.ADAM_EPS):
    G = np.asarray(G, float)
    M_new = beta1 * np.asarray(M, float) + (1 - beta1) * G
    V_new = beta2 * np.asarray(V, float) + (1 - beta2) * np.abs(G)
    U = (M_new / (1 - beta1 ** t)) / (np.sqrt(V_new / (1 - beta2 ** t)) + eps)
    return M_new, V_new, U


def himuon_shared_normalisation(U, tile, steps=5, eps=o.NS_EPS, coeffs=None):
    U = np.asarray(U, float)
    X = U / (ORIG["fro"](U) + eps)
    O = np.empty_like(U)
    for i in range(0, U.shape[0], tile):
        for j in range(0, U.shape[1], tile):
            t = X[i:i + tile, j:j + tile]
            tall = t.shape[0] > t.shape[1]
            r = _raw_iteration(t.T if tall else t, steps, coeffs)
            O[i:i + tile, j:j + tile] = r.T if tall else r
    return O


def himuon_anchored_at_the_far_corner(U, tile, steps=5, eps=o.NS_EPS, coeffs=None):
    U = np.asarray(U, float)
    return ORIG["himuon_ns"](U[::-1, ::-1], tile, steps, eps, coeffs)[::-1, ::-1].copy()


def ridge_over_tokens(Z, ridge_rel):
    Z = np.asarray(Z, float)
    return ridge_rel * float(np.sum(Z * Z)) / Z.shape[1]


def precondition_without_ridge(U, Z, ridge_rel):
    return ORIG["newton_precondition"](U, Z, 0.0)


def precondition_multiplies_instead_of_solving(U, Z, ridge_rel):
    U = np.asarray(U, float)
    Z = np.asarray(Z, float)
    S = Z @ Z.T
    S = S + ORIG["ridge_lambda"](Z, ridge_rel) * np.eye(S.shape[0])
    return U @ S


MUTATIONS = [
    ("momentum", nesterov_from_old_buffer),
    ("momentum", plain_momentum_from_old_buffer),
    ("newton_schulz", ns_sign_of_b),
    ("newton_schulz", ns_without_c),
    ("newton_schulz", ns_one_iteration_short),
    ("newton_schulz", ns_without_eps),
    ("newton_schulz", ns_spectral_normalisation),
    ("coeff_table", coefficient_table_reversed),
    ("scalar_ns", scalar_map_sign_of_b),
    ("msgn_svd", msgn_rows_and_columns_reversed),
    ("fro", fro_without_sqrt),
    ("shape_scale", shape_scale_inverted),
    ("muon_apply", muon_ignores_weight_decay),
    ("muon_apply", muon_decay_without_lr),
    ("hyperball_apply", hyperball_adds_the_step),
    ("hyperball_apply", hyperball_unnormalised_update),
    ("hyperball_apply", hyperball_ignores_radius),
    ("hyperball_apply", hyperball_without_reprojection),
    ("radial_brake_apply", brake_factors_swapped),
    ("radial_brake_apply", brake_target_from_the_new_norm),
    ("relative_update_apply", relative_update_unnormalised),
    ("adam_update", adam_without_bias_correction),
    ("adam_update", adam_second_moment_of_g),
    ("himuon_ns", himuon_shared_normalisation),
    ("himuon_ns", himuon_anchored_at_the_far_corner),
    ("ridge_lambda", ridge_over_tokens),
    ("newton_precondition", precondition_without_ridge),
    ("newton_precondition", precondition_multiplies_instead_of_solving),
]


def test_clean_oracle_passes_every_pin():
    assert failing_pins() == []


@pytest.mark.parametrize("target,mutant", MUTATIONS, ids=[m.__name__ for _, m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, target, mutant):
    monkeypatch.setattr(o, target, mutant)
    caught = failing_pins()
    assert caught, f"no pin catches {mutant.__name__} in oracle.{target}"
