"""Plain CPU fp64 oracle for the Muon / Hyperball optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or
executes this file: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or helper with the CUDA library.

Every routine works in float64 on NumPy arrays and follows the pages' update
rules in their own order.  Sources (page title, then section):

* "Muon: the orthogonalized optimizer explained through equations, intuition,
  code and results" (wpnews.pro) -- momentum recap note, Newton-Schulz section,
  the single-GPU ``newton_schulz5`` / ``Muon`` code section.
* "Fantastic Pretraining Optimizers and Where to Find Them II: Hyperball
  Optimization" (bud-325.pages.dev) -- Method section, the update
  W <- rho * Pi(W - eta * U_hat), U_hat = U~ / ||U~||_F.
* "Refactor of pre/post weight update hook functions" (NVIDIA-NeMo /
  Emerging-Optimizers PR #224) -- description of the Hyperball and RadialBrake
  hooks, the RadialBrake norm formula, and the review notes on eps and the
  zero-norm branch.
* "Hierarchical Muon: Tiled Newton-Schulz Updates" (arXiv 2606.27216) --
  abstract / core claim: the same finite NS map run independently on T x T
  tiles, then reassembled.
* "The Newton-Muon Optimizer" (arXiv 2604.01472) -- abstract: the update
  msgn(G (Z Z^T)^-1), "up to momentum and weight decay".
* The same hook PR's file list -- the RelativeUpdate hook: a pre-update scaling
  that matches the update's norm to the current weight norm.
* The Hyperball paper, Method -- Hyperball wraps any base step, Adam's
  preconditioned update among them (AdamH); Adam itself as in "Adam: A Method
  for Stochastic Optimization" (Kingma and Ba, 2014), which the pages cite.

Parity status: every public function here is pinned by ``tests/test_oracle_pins.py``
against page-printed values, closed forms, library routines or invariants.
"""
from __future__ import annotations

import numpy as np

# Quintic coefficients (a, b, c) of the Newton-Schulz map; Muon explainer,
# Newton-Schulz section and the newton_schulz5 code.
KELLER_ABC = (3.4445, -4.7750, 2.0315)
# Textbook cubic 1.5 s - 0.5 s^3 (same section), written as (a, b, c) with c = 0.
TEXTBOOK_ABC = (1.5, -0.5, 0.0)
# Second stage of the two-stage schedule named in the same section.
SETTLE_ABC = (2.0, -1.5, 0.5)

NS_EPS = 1e-7      # additive eps on ||X||_F before the first iteration (newton_schulz5 code)
HB_EPS = 1e-8      # Hyperball / RadialBrake numerical-zero threshold (PR #224 constructor default)


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def fro(x) -> float:
    """Frobenius norm, ||x||_F = sqrt(sum x_ij^2)."""
    x = _f64(x)
    return float(np.sqrt(np.sum(x * x)))


def coeff_table(steps: int, coeffs=None) -> list:
    """Per-iteration (a, b, c).  ``coeffs`` may be one triple or a list of triples."""
    if coeffs is None:
        return [KELLER_ABC] * steps
    coeffs = [tuple(float(v) for v in c) for c in np.atleast_2d(np.asarray(coeffs, dtype=np.float64))]
    if len(coeffs) == 1:
        return coeffs * steps
    if len(coeffs) != steps:
        raise ValueError("coefficient table must have one row or one row per iteration")
    return coeffs


# --------------------------------------------------------------------------
# Momentum (Muon explainer: recap note "Momentum is an exponential weighted
# average" and the Muon.step code: buf.lerp_(g, 1-mu); update = g.lerp(buf, mu)).
# --------------------------------------------------------------------------
def momentum(M, G, beta: float, nesterov: bool = True):
    """Return (M_new, U).

    M_new = beta * M + (1 - beta) * G          (EMA form of the momentum buffer)
    U     = (1 - beta) * G + beta * M_new       if nesterov (G moved toward M_new by beta)
          = M_new                                otherwise
    """
    M = _f64(M)
    G = _f64(G)
    M_new = beta * M + (1.0 - beta) * G
    U = (1.0 - beta) * G + beta * M_new if nesterov else M_new.copy()
    return M_new, U


# --------------------------------------------------------------------------
# Newton-Schulz (Muon explainer, Newton-Schulz section: the odd quintic
# phi(x) = a x + b x^3 + c x^5 applied to the matrix, i.e. to every singular value).
# --------------------------------------------------------------------------
def quintic(X, a: float, b: float, c: float):
    """The odd matrix polynomial phi(X) = a X + b (X X^T) X + c (X X^T)^2 X.

    Since (X X^T)^k X = X (X^T X)^k, phi(X) = q(X X^T) X = X q(X^T X) with the
    polynomial q(S) = a I + b S + c S^2 of a Gram matrix.  The Gram matrix of the
    shorter side is the smaller one: the left Gram X X^T when X has no more rows
    than columns, the right Gram X^T X otherwise."""
    if X.shape[0] <= X.shape[1]:
        S = X @ X.T
        return (a * np.eye(S.shape[0]) + b * S + c * (S @ S)) @ X
    S = X.T @ X
    return X @ (a * np.eye(S.shape[0]) + b * S + c * (S @ S))


def newton_schulz(G, steps: int = 5, eps: float = NS_EPS, coeffs=None):
    """Approximate msgn(G) = U V^T: scale G to (at most) unit Frobenius norm,
    X_0 = G / (||G||_F + eps), then apply the quintic ``steps`` times,
    X_{k+1} = phi_k(X_k) with the k-th (a, b, c) of the coefficient table."""
    X = _f64(G) / (fro(G) + eps)
    for a, b, c in coeff_table(steps, coeffs):
        X = quintic(X, a, b, c)
    return np.ascontiguousarray(X)


def scalar_ns(sigma, steps: int = 5, coeffs=None):
    """The scalar map sigma -> a s + b s^3 + c s^5 applied ``steps`` times (no normalisation)."""
    s = _f64(sigma)
    for a, b, c in coeff_table(steps, coeffs):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def msgn_svd(G):
    """Exact msgn(G) = U V^T from the compact SVD G = U S V^T (LAPACK)."""
    U, _, Vt = np.linalg.svd(_f64(G), full_matrices=False)
    return U @ Vt


def shape_scale(rows: int, cols: int) -> float:
    """max(1, rows/cols)^0.5 (the Muon.step code's shape scaling)."""
    return max(1.0, rows / cols) ** 0.5


# --------------------------------------------------------------------------
# Weight-update rules.
# --------------------------------------------------------------------------
def muon_apply(W, O, lr: float, weight_decay: float = 0.0):
    """Plain Muon update (Muon.step code): W <- (1 - lr wd) W - lr * max(1, m/n)^0.5 * O."""
    W = _f64(W)
    O = _f64(O)
    return (1.0 - lr * weight_decay) * W - lr * shape_scale(*W.shape) * O


def hyperball_apply(W, O, eta: float, rho: float | None, eps: float = HB_EPS):
    """Hyperball wrapper (Hyperball paper, Method): W <- rho * (W - eta U_hat) / ||W - eta U_hat||_F.

    U_hat = O / max(||O||_F, eps)  (a zero update is the zero direction).
    rho None (or <= 0) means "radius = current ||W||_F" (PR #224 Hyperball(radius=None));
    a zero current norm is then an error (ValueError, as in the PR).
    When ||W - eta U_hat||_F < eps the PR would return zero; this oracle instead keeps
    the radius: W <- rho * W / ||W||_F (the step is skipped, the direction kept).
    Returns (W_new, fallback_taken).
    """
    W = _f64(W)
    O = _f64(O)
    cur = fro(W)
    if rho is None or rho <= 0.0:
        if cur < eps:
            raise ValueError("Hyperball needs a non-zero weight norm when the radius is not fixed")
        rho = cur
    U_hat = O / max(fro(O), eps)
    V = W - eta * U_hat
    q = fro(V)
    if q < eps:
        if cur < eps:
            raise ValueError("Hyperball cannot project a zero weight onto the sphere")
        return rho * W / cur, True
    return rho * V / q, False


def radial_brake_apply(W, O, lr: float, outward: float, inward: float, eps: float = HB_EPS):
    """RadialBrake hook (PR #224): plain Muon step, then damp the change of ||w||.

    w = w_prev - lr * max(1, m/n)^0.5 * O;  delta = ||w|| - ||w_prev||;
    s = outward if delta > 0 else inward;   ||w_brake|| = ||w_prev|| + s * delta.
    w is left unscaled when ||w|| < eps.
    """
    if not (0.0 <= outward <= 1.0 and 0.0 <= inward <= 1.0):
        raise ValueError("RadialBrake factors must lie in [0, 1]")
    w_prev = _f64(W)
    w = muon_apply(w_prev, O, lr, 0.0)
    n_prev = fro(w_prev)
    n_new = fro(w)
    if n_new < eps:
        return w
    delta = n_new - n_prev
    s = outward if delta > 0 else inward
    return w * ((n_prev + s * delta) / n_new)


def relative_update_apply(W, O, lr: float, weight_decay: float = 0.0, eps: float = HB_EPS):
    """RelativeUpdate hook (PR #224): before the Muon update is applied, rescale it to the
    Frobenius norm of the current weight.  The update max(1, m/n)^0.5 * O has direction
    O / ||O||, so its shape factor cancels:
        W <- (1 - lr wd) W - lr * ||W||_F * O / max(||O||_F, eps)
    (a zero update stays zero, as in the hooks' eps clamp)."""
    W = _f64(W)
    O = _f64(O)
    return (1.0 - lr * weight_decay) * W - lr * fro(W) * O / max(fro(O), eps)


# --------------------------------------------------------------------------
# Adam (Kingma and Ba, 2014), the base step of AdamH (Hyperball paper, Method).
# --------------------------------------------------------------------------
ADAM_BETA1 = 0.9
ADAM_BETA2 = 0.999
ADAM_EPS = 1e-8


def adam_update(M, V, G, t: int, beta1: float = ADAM_BETA1, beta2: float = ADAM_BETA2, eps: float = ADAM_EPS):
    """Moments and the bias-corrected Adam direction of step t (t = 1 is the first step):
        M <- beta1 M + (1 - beta1) G;   V <- beta2 V + (1 - beta2) G^2;
        U~ = (M / (1 - beta1^t)) / (sqrt(V / (1 - beta2^t)) + eps).
    Returns (M_new, V_new, U~)."""
    if t < 1:
        raise ValueError("Adam steps count from 1")
    M = _f64(M)
    V = _f64(V)
    G = _f64(G)
    M_new = beta1 * M + (1.0 - beta1) * G
    V_new = beta2 * V + (1.0 - beta2) * G * G
    m_hat = M_new / (1.0 - beta1 ** t)
    v_hat = V_new / (1.0 - beta2 ** t)
    return M_new, V_new, m_hat / (np.sqrt(v_hat) + eps)


# --------------------------------------------------------------------------
# Hierarchical Muon (arXiv 2606.27216, abstract / core claim).
# --------------------------------------------------------------------------
def himuon_ns(U, tile: int, steps: int = 5, eps: float = NS_EPS, coeffs=None):
    """Partition U into tile x tile blocks anchored at (0, 0) (edge blocks are the
    remainder), run the same finite NS map on each block independently, reassemble."""
    U = _f64(U)
    O = np.empty_like(U)
    m, n = U.shape
    for i in range(0, m, tile):
        for j in range(0, n, tile):
            O[i:i + tile, j:j + tile] = newton_schulz(U[i:i + tile, j:j + tile], steps, eps, coeffs)
    return O


# --------------------------------------------------------------------------
# Newton-Muon (arXiv 2604.01472, abstract): msgn(G (Z Z^T)^-1), here with a ridge.
# --------------------------------------------------------------------------
def ridge_lambda(Z, ridge_rel: float) -> float:
    """lambda = ridge_rel * tr(Z Z^T) / d_in  (tr(Z Z^T) = ||Z||_F^2)."""
    Z = _f64(Z)
    return ridge_rel * float(np.sum(Z * Z)) / Z.shape[0]


def newton_precondition(U, Z, ridge_rel: float):
    """P = U (Z Z^T + lambda I)^-1, by a plain linear solve of P S = U (S symmetric)."""
    U = _f64(U)
    Z = _f64(Z)
    S = Z @ Z.T + ridge_lambda(Z, ridge_rel) * np.eye(Z.shape[0])
    return np.linalg.solve(S, U.T).T


# --------------------------------------------------------------------------
# Whole steps, in the pages' order: momentum -> (precondition) -> NS -> hook.
# --------------------------------------------------------------------------
def muon_step(W, G, M, *, beta=0.95, nesterov=True, steps=5, ns_eps=NS_EPS, coeffs=None,
              lr=0.02, weight_decay=0.0):
    M_new, U = momentum(M, G, beta, nesterov)
    O = newton_schulz(U, steps, ns_eps, coeffs)
    return muon_apply(W, O, lr, weight_decay), M_new, O


def hyperball_step(W, G, M, *, eta, rho, beta=0.95, nesterov=True, steps=5, ns_eps=NS_EPS,
                   coeffs=None, hb_eps=HB_EPS):
    M_new, U = momentum(M, G, beta, nesterov)
    O = newton_schulz(U, steps, ns_eps, coeffs)
    W_new, fb = hyperball_apply(W, O, eta, rho, hb_eps)
    return W_new, M_new, O, fb


def radial_brake_step(W, G, M, *, lr, outward, inward, beta=0.95, nesterov=True, steps=5,
                      ns_eps=NS_EPS, coeffs=None, hb_eps=HB_EPS):
    M_new, U = momentum(M, G, beta, nesterov)
    O = newton_schulz(U, steps, ns_eps, coeffs)
    return radial_brake_apply(W, O, lr, outward, inward, hb_eps), M_new, O


def himuon_step(W, G, M, *, tile, eta, rho, beta=0.95, nesterov=True, steps=5, ns_eps=NS_EPS,
                coeffs=None, hb_eps=HB_EPS):
    M_new, U = momentum(M, G, beta, nesterov)
    O = himuon_ns(U, tile, steps, ns_eps, coeffs)
    W_new, fb = hyperball_apply(W, O, eta, rho, hb_eps)
    return W_new, M_new, O, fb


def newton_muon_step(W, G, M, Z, *, ridge_rel, eta, rho, beta=0.95, nesterov=True, steps=5,
                     ns_eps=NS_EPS, coeffs=None, hb_eps=HB_EPS):
    M_new, U = momentum(M, G, beta, nesterov)
    P = newton_precondition(U, Z, ridge_rel)
    O = newton_schulz(P, steps, ns_eps, coeffs)
    W_new, fb = hyperball_apply(W, O, eta, rho, hb_eps)
    return W_new, M_new, O, fb


def relative_update_step(W, G, M, *, lr, weight_decay=0.0, beta=0.95, nesterov=True, steps=5,
                         ns_eps=NS_EPS, coeffs=None, hb_eps=HB_EPS):
    M_new, U = momentum(M, G, beta, nesterov)
    O = newton_schulz(U, steps, ns_eps, coeffs)
    return relative_update_apply(W, O, lr, weight_decay, hb_eps), M_new, O


def adamh_step(W, G, M, V, *, t, eta, rho, beta1=ADAM_BETA1, beta2=ADAM_BETA2, adam_eps=ADAM_EPS,
               hb_eps=HB_EPS):
    """AdamH: the Adam direction of step t, wrapped by Hyperball.
    Returns (W_new, M_new, V_new, U~, fallback_taken)."""
    M_new, V_new, U = adam_update(M, V, G, t, beta1, beta2, adam_eps)
    W_new, fb = hyperball_apply(W, U, eta, rho, hb_eps)
    return W_new, M_new, V_new, U, fb
