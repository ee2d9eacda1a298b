"""Plain float64 spectral diagnostics and spectral cap -- TEST INFRASTRUCTURE ONLY.

* Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
  Muon lowers the condition number of the projection it trains; the
  practitioner notes (section 7.2) check the top singular value of the state
  matrices periodically.  power_iteration() is the plainest estimate of the
  top singular triplet, stable_rank() the isotropy measure beside it.
* An Isotropy-Preserving Spectral Cap for Muon, summary and "unified theory":
  each update has the direction that contributes most to the growth of the
  top eigenvalue removed, while learning continues through the other
  directions.  READING: with (u, v) the top singular pair of the pre-step W,
  the first-order growth of sigma_max under W - eta O is -eta u^T O v, so the
  cap removes that component: O <- O - (u^T O v) u v^T.
"""
from __future__ import annotations

import numpy as np

from .muon_oracle import (apply_update, frobenius_norm, momentum_update, nesterov_lookahead, orthogonalize,
                          shape_scale, wide_view)


def power_iteration(W, v0, iters: int):
    """k steps of u = W v / |W v|, v = W^T u / |W^T u|, sigma = |W^T u| from the start vector v0.

    Returns (u, v, sigma).  A zero W returns zero vectors and sigma 0.
    """
    W = np.asarray(W, np.float64)
    v = np.asarray(v0, np.float64)
    v = v / np.linalg.norm(v)
    u = np.zeros(W.shape[0])
    sigma = 0.0
    for _ in range(iters):
        u = W @ v
        nu = np.linalg.norm(u)
        if nu == 0.0:
            return np.zeros(W.shape[0]), np.zeros(W.shape[1]), 0.0
        u = u / nu
        v = W.T @ u
        sigma = float(np.linalg.norm(v))
        if sigma == 0.0:
            return u, np.zeros(W.shape[1]), 0.0
        v = v / sigma
    return u, v, sigma


def min_singular_shifted(W, y0, sigma_max: float, iters: int):
    """Smallest singular value of W's wide view X (m = min(rows, cols) rows) by shifted power iteration.

    With s = sigma_max^2, the largest eigenvalue of s I - X X^T is s - sigma_min^2,
    so `iters` steps of y <- (s y - X (X^T y)) / |.| turn y toward the bottom left
    singular vector of X; the estimate is the Rayleigh value |X^T y|, which is
    >= sigma_min for every unit y.  Returns (y, sigma_min); kappa = sigma_max /
    sigma_min.  READING: the pages report the condition number falling under
    Muon without saying how it is computed; this is the plainest iteration that
    needs only products with W.
    """
    X, _ = wide_view(np.asarray(W, np.float64))
    s = float(sigma_max) ** 2
    y = np.asarray(y0, np.float64)
    y = y / np.linalg.norm(y)
    for _ in range(iters):
        y = s * y - X @ (X.T @ y)
        n = np.linalg.norm(y)
        if n == 0.0:
            break
        y = y / n
    return y, float(np.linalg.norm(X.T @ y))


def stable_rank(W, sigma_max: float) -> float:
    """||W||_F^2 / sigma_max^2 (1 for a rank-one matrix, min(rows, cols) for an isotropic one)."""
    return frobenius_norm(W) ** 2 / sigma_max ** 2


def spectral_cap(O, u, v):
    """O - (u^T O v) u v^T: the update without its first-order push on sigma_max(W)."""
    O = np.asarray(O, np.float64)
    alpha = float(u @ O @ v)
    return O - alpha * np.outer(u, v), alpha


def muon_step_capped(W, G, M, coeffs, u, v, lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7,
                     nesterov=True, scale_mode=0):
    """muon_step with the orthogonalised update capped against the (u, v) direction of the pre-step W."""
    M_new = momentum_update(M, G, beta)
    U = nesterov_lookahead(G, M_new, beta) if nesterov else M_new
    O, nu = orthogonalize(U, coeffs, eps)
    Oc, alpha = spectral_cap(O, u, v)
    rows, cols = np.shape(W)
    return dict(W=apply_update(W, Oc, lr, weight_decay, shape_scale(rows, cols, scale_mode)), M=M_new,
                O=Oc, alpha=alpha, nu=nu)
