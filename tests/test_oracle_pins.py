"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test names the passage it follows.  None of them recomputes an oracle
formula the oracle's own way: they use values printed on the pages
(tests/golden/page_values.json), LAPACK (SVD, Cholesky), closed forms of
multi-step processes, and invariances.
"""
import json
import math
import pathlib

import numpy as np
import pytest
import scipy.linalg

from oracle import nshb_oracle as o

GOLD = json.loads((pathlib.Path(__file__).parent / "golden" / "page_values.json").read_text())


def _orth(rng, n, k):
    q, _ = np.linalg.qr(rng.standard_normal((n, k)))
    return q


def _with_spectrum(rng, m, n, sigma):
    k = len(sigma)
    return (_orth(rng, m, k) * np.asarray(sigma)) @ _orth(rng, n, k).T


# ---------------------------------------------------------------- scalar map
def test_textbook_cubic_from_001():
    g = GOLD["textbook_cubic_from_0.01_after_5"]
    assert abs(o.scalar_ns(0.01, 5, o.TEXTBOOK_ABC) - g["value"]) <= g["abs_tol"]


def test_quintic_slope_at_zero():
    g = GOLD["slope_at_zero"]
    h = 1e-9
    assert abs(o.scalar_ns(h, 1) / h - g["value"]) <= g["abs_tol"]


def test_quintic_band_on_scalar_map():
    g = GOLD["band"]
    x = np.linspace(g["in_lo"], g["in_hi"], 200001)
    y = o.scalar_ns(x, 5)
    assert abs(y.min() - g["out_lo"]) <= g["abs_tol"]
    assert abs(y.max() - g["out_hi"]) <= g["abs_tol"]


# ---------------------------------------------------- matrix NS vs the pages
def test_five_direction_example():
    g = GOLD["five_directions"]
    rng = np.random.default_rng(1)
    M = _with_spectrum(rng, 5, 5, g["sigma"])
    assert abs(o.fro(M) - g["frobenius_norm"]) <= g["frobenius_abs_tol"]
    entering = np.linalg.svd(M / (o.fro(M) + o.NS_EPS), compute_uv=False)
    assert np.allclose(entering, g["entering"], rtol=g["entering_rel_tol"])
    s_out = np.linalg.svd(o.newton_schulz(M, 5), compute_uv=False)
    assert abs(s_out.min() - g["out_min"]) <= g["out_abs_tol"]
    assert abs(s_out.max() - g["out_max"]) <= g["out_abs_tol"]
    assert abs(max(g["sigma"]) / min(g["sigma"]) - g["cond_in"]) < 1e-9
    assert abs(s_out.max() / s_out.min() - g["cond_out"]) <= g["cond_out_abs_tol"]


def test_two_by_two_example():
    g = GOLD["two_by_two"]
    M = _with_spectrum(np.random.default_rng(2), 2, 2, g["sigma"])
    s_out = np.sort(np.linalg.svd(o.newton_schulz(M, 5), compute_uv=False))
    assert np.all(np.abs(s_out - np.array(g["out"])) <= g["abs_tol"])


@pytest.mark.parametrize("shape", [(7, 4), (4, 7), (5, 5), (1, 6), (6, 1), (9, 3)])
def test_ns_svd_identity(shape):
    """NS_K(M) = U phi^K(S / (||M|| + eps)) V^T in exact arithmetic (odd polynomial of X)."""
    rng = np.random.default_rng(hash(shape) % 2**32)
    M = rng.standard_normal(shape)
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    expect = (U * o.scalar_ns(S / (np.sqrt(np.sum(S ** 2)) + o.NS_EPS), 5)) @ Vt
    assert np.allclose(o.newton_schulz(M, 5), expect, atol=1e-12, rtol=0)


def test_ns_within_band_of_msgn():
    """||NS(M) - U V^T||_2 <= max |phi^5(x) - 1| over the normalised singular values."""
    rng = np.random.default_rng(3)
    sig = np.geomspace(0.02, 1.0, 6)
    M = _with_spectrum(rng, 8, 6, sig)
    err = np.linalg.norm(o.newton_schulz(M, 5) - o.msgn_svd(M), 2)
    bound = np.max(np.abs(o.scalar_ns(sig / np.sqrt(np.sum(sig ** 2)), 5) - 1.0))
    assert err <= bound + 1e-12


def test_textbook_cubic_converges_to_msgn():
    rng = np.random.default_rng(4)
    M = _with_spectrum(rng, 6, 9, np.linspace(0.3, 1.0, 6))
    assert np.allclose(o.newton_schulz(M, 60, coeffs=o.TEXTBOOK_ABC), o.msgn_svd(M), atol=1e-10)


def test_ns_equivariances():
    rng = np.random.default_rng(5)
    M = rng.standard_normal((6, 10))
    Q = _orth(rng, 6, 6)
    R = _orth(rng, 10, 10)
    O = o.newton_schulz(M)
    assert np.allclose(o.newton_schulz(Q @ M @ R), Q @ O @ R, atol=1e-11)
    assert np.allclose(o.newton_schulz(M.T), O.T, atol=1e-12)
    assert np.allclose(o.newton_schulz(37.5 * M), O, atol=1e-7)


def test_ns_zero_and_per_iteration_table():
    assert np.all(o.newton_schulz(np.zeros((4, 3))) == 0)
    rng = np.random.default_rng(6)
    M = rng.standard_normal((5, 8))
    table = [o.KELLER_ABC] * 3 + [o.SETTLE_ABC] * 2
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    s = S / (np.sqrt(np.sum(S ** 2)) + o.NS_EPS)
    s = o.scalar_ns(o.scalar_ns(s, 3, o.KELLER_ABC), 2, o.SETTLE_ABC)
    assert np.allclose(o.newton_schulz(M, 5, coeffs=table), (U * s) @ Vt, atol=1e-12)


# --------------------------------------------------------------- momentum
def test_momentum_closed_form_constant_gradient():
    """Constant G from M0 = 0: M_t = (1 - b^t) G, Nesterov U_t = (1 - b^(t+1)) G."""
    rng = np.random.default_rng(7)
    G = rng.standard_normal((3, 4))
    beta = 0.95
    M = np.zeros_like(G)
    for t in range(1, 8):
        M, U = o.momentum(M, G, beta, True)
        assert np.allclose(M, (1 - beta ** t) * G, atol=1e-14)
        assert np.allclose(U, (1 - beta ** (t + 1)) * G, atol=1e-14)
        _, U_plain = o.momentum(M * 0 + M, G * 0, 1.0, False)
        assert np.array_equal(U_plain, M)


def test_plain_momentum_closed_form_constant_gradient():
    """Without Nesterov the update is the new buffer itself: U_t = M_t = (1 - b^t) G for a
    constant G from M0 = 0 (an update taken from the old buffer would give (1 - b^(t-1)) G)."""
    rng = np.random.default_rng(9)
    G = rng.standard_normal((4, 3))
    beta = 0.9
    M = np.zeros_like(G)
    for t in range(1, 6):
        M, U = o.momentum(M, G, beta, False)
        assert np.allclose(U, (1 - beta ** t) * G, atol=1e-14)
        assert np.array_equal(U, M)


def test_sum_form_momentum_gives_same_update():
    """Keller's sum form M' = b M' + G is (1-b)^-1 times the EMA, so NS agrees (scale invariance)."""
    rng = np.random.default_rng(8)
    beta = 0.9
    M = np.zeros((5, 7))
    Ms = np.zeros((5, 7))
    for _ in range(4):
        G = rng.standard_normal((5, 7))
        M, U = o.momentum(M, G, beta, True)
        Ms = beta * Ms + G
        U_sum = G + beta * Ms
        assert np.allclose(o.newton_schulz(U), o.newton_schulz(U_sum), atol=1e-6)


# ------------------------------------------------------------- muon apply
def test_noop_is_bit_exact():
    rng = np.random.default_rng(9)
    W = rng.standard_normal((5, 7))
    O = rng.standard_normal((5, 7))
    assert np.array_equal(o.muon_apply(W, O, 0.0, 0.0), W)


def test_weight_decay_geometric():
    """G = 0 gives U = 0, O = 0, so W_t = (1 - lr wd)^t W_0."""
    rng = np.random.default_rng(10)
    W0 = rng.standard_normal((4, 6))
    W, M = W0.copy(), np.zeros_like(W0)
    for _ in range(5):
        W, M, O = o.muon_step(W, np.zeros_like(W0), M, lr=0.1, weight_decay=0.5)
        assert np.all(O == 0)
    assert np.allclose(W, 0.95 ** 5 * W0, atol=1e-14)


@pytest.mark.parametrize("shape", [(12, 5), (5, 12), (7, 7)])
def test_shape_scaling_gives_rms_one_over_sqrt_cols(shape):
    """With an exact msgn (textbook cubic run to convergence), the shape-scaled update
    has RMS 1/sqrt(cols) for tall, wide and square full-rank matrices."""
    rng = np.random.default_rng(11)
    G = _with_spectrum(rng, *shape, np.linspace(0.4, 1.0, min(shape)))
    M0 = np.zeros(shape)
    W0 = np.zeros(shape)
    W, _, _ = o.muon_step(W0, G, M0, beta=0.0, nesterov=False, steps=60, coeffs=o.TEXTBOOK_ABC, lr=1.0)
    rms = np.sqrt(np.mean(W ** 2))
    assert abs(rms - 1 / math.sqrt(shape[1])) < 1e-9


# -------------------------------------------------------------- hyperball
def test_hyperball_radius_and_angle():
    """||W_new|| = rho; when U_hat is orthogonal to W the rotation angle is atan(eta / rho)."""
    rng = np.random.default_rng(12)
    W = rng.standard_normal((6, 8))
    rho = o.fro(W)
    O = rng.standard_normal((6, 8))
    O -= (np.sum(O * W) / np.sum(W * W)) * W          # make O orthogonal to W
    eta = 0.37
    W_new, fb = o.hyperball_apply(W, 3.0 * O, eta, rho)
    assert not fb
    assert abs(o.fro(W_new) - rho) < 1e-12
    cosang = np.sum(W_new * W) / (o.fro(W_new) * o.fro(W))
    assert abs(math.acos(min(1.0, cosang)) - math.atan(eta / rho)) < 1e-12


def test_hyperball_fixed_radius_and_current_radius():
    rng = np.random.default_rng(13)
    W = rng.standard_normal((3, 5))
    O = rng.standard_normal((3, 5))
    W1, _ = o.hyperball_apply(W, O, 0.1, 2.5)
    assert abs(o.fro(W1) - 2.5) < 1e-12
    W2, _ = o.hyperball_apply(W, O, 0.1, None)
    assert abs(o.fro(W2) - o.fro(W)) < 1e-12
    with pytest.raises(ValueError):
        o.hyperball_apply(np.zeros((3, 5)), O, 0.1, None)


def test_hyperball_zero_update_keeps_direction():
    rng = np.random.default_rng(14)
    W = rng.standard_normal((4, 4))
    W1, fb = o.hyperball_apply(W, np.zeros((4, 4)), 0.2, 3.0)
    assert not fb
    assert np.allclose(W1, 3.0 * W / o.fro(W), atol=1e-14)


def test_hyperball_exactly_cancelling_update_keeps_radius():
    """rho = eta and W = eta U_hat: W - eta U_hat = 0; the radius must still be rho."""
    rng = np.random.default_rng(15)
    O = rng.standard_normal((5, 7))
    eta = 0.02
    W = eta * (O / o.fro(O))
    W1, fb = o.hyperball_apply(W, O, eta, eta)
    assert fb
    assert abs(o.fro(W1) - eta) < 1e-15
    assert np.allclose(W1 / o.fro(W1), O / o.fro(O), atol=1e-12)


def test_hyperball_step_keeps_radius_over_steps():
    rng = np.random.default_rng(16)
    W = 0.02 * rng.standard_normal((16, 24))
    rho = o.fro(W)
    M = np.zeros_like(W)
    for t in range(10):
        W, M, O, fb = o.hyperball_step(W, 1e-2 * rng.standard_normal(W.shape), M, eta=0.02, rho=rho)
        assert abs(o.fro(W) - rho) / rho < 1e-13 and not fb


# ------------------------------------------------------------ radial brake
def test_radial_brake_page_targets():
    g = GOLD["radial_brake_targets"]
    lr = 0.5
    w_prev = np.array([[3.0, 4.0]])                      # ||w_prev|| = 5
    O = -np.array([[3.0, 4.0]]) / lr                     # w = [6, 8], ||w|| = 10, outward
    w = o.radial_brake_apply(w_prev, O, lr, 0.5, 1.0)
    assert o.fro(w) == g["outward_target"]
    w_prev = np.array([[6.0, 8.0]])                      # ||w_prev|| = 10
    O = np.array([[1.2, 1.6]]) / lr                      # w = [4.8, 6.4], ||w|| = 8, inward
    w = o.radial_brake_apply(w_prev, O, lr, 1.0, 0.5)
    assert abs(o.fro(w) - g["inward_target"]) < 1e-12


def test_radial_brake_limits():
    rng = np.random.default_rng(17)
    W = rng.standard_normal((6, 3))
    O = rng.standard_normal((6, 3))
    plain = o.muon_apply(W, O, 0.3)
    assert np.allclose(o.radial_brake_apply(W, O, 0.3, 1.0, 1.0), plain, atol=1e-14)
    held = o.radial_brake_apply(W, O, 0.3, 0.0, 0.0)
    assert abs(o.fro(held) - o.fro(W)) < 1e-12
    assert np.allclose(held / o.fro(held), plain / o.fro(plain), atol=1e-14)
    with pytest.raises(ValueError):
        o.radial_brake_apply(W, O, 0.3, 1.5, 1.0)


# ---------------------------------------------------------------- HiMuon
def test_himuon_large_tile_is_full_muon():
    rng = np.random.default_rng(18)
    U = rng.standard_normal((12, 20))
    assert np.array_equal(o.himuon_ns(U, 20), o.newton_schulz(U))
    assert np.array_equal(o.himuon_ns(U, 64), o.newton_schulz(U))


def test_himuon_tile_is_svd_map_of_tile_alone():
    """Each output tile equals U_t phi^5(S_t/||tile||) V_t^T of its own input tile (LAPACK),
    including the ragged edge tiles, with the grid anchored at (0, 0)."""
    rng = np.random.default_rng(19)
    U = rng.standard_normal((10, 13))
    T = 4
    O = o.himuon_ns(U, T)
    for i in range(0, 10, T):
        for j in range(0, 13, T):
            t = U[i:i + T, j:j + T]
            u, s, vt = np.linalg.svd(t, full_matrices=False)
            expect = (u * o.scalar_ns(s / (np.sqrt(np.sum(s ** 2)) + o.NS_EPS), 5)) @ vt
            assert np.allclose(O[i:i + T, j:j + T], expect, atol=1e-12)


# ------------------------------------------------------------ Newton-Muon
def test_newton_precondition_solves_and_matches_cholesky():
    rng = np.random.default_rng(20)
    U = rng.standard_normal((5, 6))
    Z = rng.standard_normal((6, 40)) * np.exp(rng.uniform(-1, 1, (6, 1)))
    P = o.newton_precondition(U, Z, 1e-3)
    lam = 1e-3 * np.trace(Z @ Z.T) / 6
    S = Z @ Z.T + lam * np.eye(6)
    assert np.linalg.norm(P @ S - U) / np.linalg.norm(U) < 1e-12
    c = scipy.linalg.cho_factor(S, lower=True)
    assert np.allclose(P, scipy.linalg.cho_solve(c, U.T).T, atol=1e-12)


def test_newton_muon_isotropic_input_is_muon():
    """Z Z^T = c I: the preconditioner is a positive scalar, so msgn is unchanged."""
    rng = np.random.default_rng(21)
    U = rng.standard_normal((4, 6))
    Z = 3.0 * _orth(rng, 50, 6).T                      # 6 x 50, orthonormal rows times 3
    P = o.newton_precondition(U, Z, 1e-3)
    assert np.allclose(P * (9.0 + 1e-3 * 9.0), U, atol=1e-12)
    assert np.allclose(o.newton_schulz(P), o.newton_schulz(U), atol=1e-6)


# ------------------------------------------------------------------ RelativeUpdate hook
def test_relative_update_step_length_is_lr_times_weight_norm():
    """The hook matches the update's norm to ||W||: with wd = 0 the step W - W_new has
    Frobenius norm lr * ||W|| exactly and points along O, whatever ||O|| and the shape."""
    rng = np.random.default_rng(41)
    for shape in [(6, 9), (9, 6), (5, 5)]:
        W = rng.standard_normal(shape)
        O = 7.5 * rng.standard_normal(shape)
        Wn = o.relative_update_apply(W, O, lr=0.03)
        step = W - Wn
        assert abs(o.fro(step) - 0.03 * o.fro(W)) <= 1e-14 * o.fro(W)
        cos = float(np.sum(step * O)) / (o.fro(step) * o.fro(O))
        assert abs(cos - 1.0) <= 1e-14


def test_relative_update_zero_update_and_weight_decay():
    rng = np.random.default_rng(42)
    W = rng.standard_normal((4, 7))
    assert np.array_equal(o.relative_update_apply(W, np.zeros_like(W), lr=0.1), W)
    O = rng.standard_normal((4, 7))
    d = o.relative_update_apply(W, O, lr=0.1, weight_decay=0.2) - o.relative_update_apply(W, O, lr=0.1)
    assert np.allclose(d, -0.1 * 0.2 * W, rtol=0, atol=1e-15)


# ------------------------------------------------------------------ Adam / AdamH
def test_adam_first_step_from_zero_state_is_g_over_abs_g():
    """Bias correction makes step 1 exact: m_hat = g, v_hat = g^2, so U~ = g / (|g| + eps)."""
    rng = np.random.default_rng(43)
    G = rng.standard_normal((5, 8)) * 1e-3
    Mn, Vn, U = o.adam_update(np.zeros_like(G), np.zeros_like(G), G, 1)
    assert np.allclose(Mn, 0.1 * G, rtol=1e-13, atol=0)        # 1 - 0.9 and 1 - 0.999 in fp64
    assert np.allclose(Vn, 0.001 * G * G, rtol=1e-13, atol=0)
    assert np.allclose(U, G / (np.abs(G) + 1e-8), rtol=1e-12, atol=0)


def test_adam_constant_gradient_keeps_the_first_direction():
    """With a constant gradient the corrected moments stay m_hat = g, v_hat = g^2 at every t."""
    G = np.array([[2.0, -0.5], [1e-3, -4.0]])
    M = np.zeros_like(G)
    V = np.zeros_like(G)
    for t in range(1, 8):
        M, V, U = o.adam_update(M, V, G, t)
        assert np.allclose(U, G / (np.abs(G) + 1e-8), rtol=1e-12, atol=0), t


def test_adam_two_steps_by_hand():
    """g = 1 then g = -1 from zero state: m2 = -0.01, v2 = 0.001999, so m_hat = -0.01 / 0.19
    = -1/19 and v_hat = 0.001999 / (1 - 0.999^2) = 1: U~2 = -(1/19) / (1 + 1e-8)."""
    M, V, U1 = o.adam_update(np.zeros(1), np.zeros(1), np.ones(1), 1)
    assert abs(U1[0] - 1.0 / (1.0 + 1e-8)) <= 1e-15
    M, V, U2 = o.adam_update(M, V, -np.ones(1), 2)
    assert abs(M[0] + 0.01) <= 1e-17 and abs(V[0] - 0.001999) <= 1e-17
    assert abs(U2[0] + (1.0 / 19.0) / (1.0 + 1e-8)) <= 1e-14


def test_adam_without_averaging_is_elementwise_sign():
    """beta1 = beta2 = 0: U~ = g / (|g| + eps), the sign of g up to eps, for any history."""
    rng = np.random.default_rng(44)
    G = rng.standard_normal((3, 4))
    _, _, U = o.adam_update(rng.standard_normal((3, 4)), rng.random((3, 4)), G, 5, beta1=0.0, beta2=0.0)
    assert np.allclose(U, G / (np.abs(G) + 1e-8), rtol=1e-12, atol=0)


def test_adamh_step_lands_on_the_sphere_along_the_adam_direction():
    rng = np.random.default_rng(45)
    W = 0.02 * rng.standard_normal((16, 24))
    G = 1e-3 * rng.standard_normal((16, 24))
    rho = o.fro(W)
    Wn, Mn, Vn, U, fb = o.adamh_step(W, G, np.zeros_like(W), np.zeros_like(W), t=1, eta=0.02, rho=rho)
    assert not fb
    assert abs(o.fro(Wn) - rho) <= 1e-14 * rho
    # W_new is W - eta * U / ||U|| rescaled: undo the scale and compare the step
    V = W - 0.02 * U / o.fro(U)
    assert np.allclose(Wn, rho * V / o.fro(V), rtol=0, atol=1e-15)
    # first step: U~ = sign(G) up to eps / |g|, so the unit direction has equal-magnitude entries
    tol = 4e-8 / float(np.min(np.abs(G)))
    assert np.allclose(np.abs(U / o.fro(U)), 1.0 / np.sqrt(U.size), rtol=tol, atol=0)
