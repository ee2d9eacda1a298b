"""Plain float64 NumPy restatement of the Muon step -- TEST INFRASTRUCTURE ONLY.

Sources (by page title and section):
  * Muon Meets Mamba: Spectral Optimization for State Space Models (arXiv
    2608.03941), abstract: Muon orthogonalises the update to each weight matrix
    with a Newton-Schulz iteration (steepest descent under the spectral norm);
    it is applied per weight group (input / output projection) of Mamba-2 130M.
  * MuonSSM: Orthogonalizing State Space Models, section "Newton-Schulz
    lightweight orthogonalisation": the iteration needs no explicit SVD; section
    "convergence and complexity": its matrix products are a constant-factor cost.
  * An Isotropy-Preserving Spectral Cap for Muon, section "unified theory": the
    update is a matrix-sign step, so its size does not shrink with 1/||W||_F.

The pages print no formula for the step.  The step order used here -- momentum
with a Nesterov look-ahead, Frobenius normalisation, k iterations of
X <- aX + (bA + cA^2)X with A = XX^T on the wide orientation, a shape scale and
decoupled weight decay -- is the problem statement this library implements;
each open choice is marked READING below.

No blocking, fusion or reordering: every step is the definition written out,
with NumPy's matmul as the only library primitive.
"""
from __future__ import annotations

import math

import numpy as np

# READING: the pages give no coefficients.  Cubic (1.5, -0.5, 0) is the classic
# Newton-Schulz polar iteration (fixed point sigma = 1); the quintic triple is
# the widely used Muon default.  Both are parameters everywhere.
CUBIC = (1.5, -0.5, 0.0)
QUINTIC = (3.4445, -4.7750, 2.0315)

SCALE_SQRT_RATIO = 0  # sqrt(max(1, rows/cols))
SCALE_NONE = 1        # 1
SCALE_RMS_MATCH = 2   # 0.2 * sqrt(max(rows, cols))


def momentum_update(M: np.ndarray, G: np.ndarray, beta: float) -> np.ndarray:
    """M <- beta*M + G (heavy-ball buffer, SGD convention).

    READING: the pages name momentum but not its convention.  The EMA form
    (M <- beta*M + (1-beta)*G) scales every later quantity by (1-beta), which
    the Frobenius normalisation removes, so the orthogonalised update is the
    same; only the stored buffer differs.
    """
    return beta * np.asarray(M, np.float64) + np.asarray(G, np.float64)


def nesterov_lookahead(G: np.ndarray, M_new: np.ndarray, beta: float) -> np.ndarray:
    """U = G + beta*M_new, the Nesterov look-ahead taken with the updated buffer."""
    return np.asarray(G, np.float64) + beta * M_new


def frobenius_norm(U: np.ndarray) -> float:
    """||U||_F = sqrt(sum of squared entries)."""
    U = np.asarray(U, np.float64)
    return float(np.sqrt(np.sum(U * U)))


def normalize(U: np.ndarray, eps: float):
    """X0 = U / (||U||_F + eps); returns (X0, ||U||_F).

    READING: eps is added to the norm (not inside the square root), so an
    all-zero U gives X0 = 0 and a zero update.
    """
    nu = frobenius_norm(U)
    return np.asarray(U, np.float64) / (nu + eps), nu


def wide_view(X: np.ndarray):
    """Return (X or X^T, transposed?) so that rows <= cols.

    READING: transpose iff rows > cols; a square matrix is not transposed.  On
    the wide view A = X X^T is the small min(rows, cols)-square Gram matrix.
    """
    X = np.asarray(X, np.float64)
    if X.shape[0] > X.shape[1]:
        return X.T, True
    return X, False


def newton_schulz(X: np.ndarray, coeffs) -> np.ndarray:
    """k Newton-Schulz steps on a wide X: A = X X^T, B = b A + c A A, X <- a X + B X.

    `coeffs` is a sequence of (a, b, c), one triple per iteration (k = len).
    Every iterate equals U p(S) V^T for X = U S V^T with p(s) = a s + b s^3 + c s^5,
    which is what the SVD pin checks.
    """
    X = np.asarray(X, np.float64)
    for (a, b, c) in coeffs:
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X


def orthogonalize(U: np.ndarray, coeffs, eps: float = 1e-7):
    """Normalise, orient wide, iterate, orient back.  Returns (O, ||U||_F)."""
    X0, nu = normalize(U, eps)
    Xw, transposed = wide_view(X0)
    Xk = newton_schulz(Xw, coeffs)
    return (Xk.T if transposed else Xk), nu


def shape_scale(rows: int, cols: int, mode: int = SCALE_SQRT_RATIO) -> float:
    """Scale applied to the orthogonalised update of a rows x cols matrix.

    READING: the pages only say the step is orthogonalised; the default
    sqrt(max(1, rows/cols)) keeps the per-entry RMS of a tall matrix's update
    equal to that of a wide one.  0.2*sqrt(max(rows, cols)) and 1 are selectable.
    """
    if mode == SCALE_SQRT_RATIO:
        return math.sqrt(max(1.0, rows / cols))
    if mode == SCALE_NONE:
        return 1.0
    if mode == SCALE_RMS_MATCH:
        return 0.2 * math.sqrt(max(rows, cols))
    raise ValueError(f"unknown scale mode {mode}")


def apply_update(W: np.ndarray, O: np.ndarray, lr: float, weight_decay: float, scale: float) -> np.ndarray:
    """W <- W (1 - lr*wd) - lr*scale*O: decoupled weight decay taken from the pre-step W."""
    W = np.asarray(W, np.float64)
    return W * (1.0 - lr * weight_decay) - lr * scale * np.asarray(O, np.float64)


def muon_step(W, G, M, coeffs, lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7,
              nesterov=True, scale_mode=SCALE_SQRT_RATIO):
    """One Muon step for one matrix.  Returns dict(W, M, O, nu, finite).

    Order: M <- beta M + G; U = G + beta M (or U = M without Nesterov);
    O = NS_k(U / (||U||_F + eps)) on the wide view; W <- W(1 - lr wd) - lr s O.
    READING (non-finite norm): the buffer keeps its update, W is left unchanged
    and the matrix is reported as non-finite.
    """
    M_new = momentum_update(M, G, beta)
    U = nesterov_lookahead(G, M_new, beta) if nesterov else M_new
    nu = frobenius_norm(U)
    if not np.isfinite(nu):
        return dict(W=np.asarray(W, np.float64), M=M_new, O=None, nu=nu, finite=False)
    O, _ = orthogonalize(U, coeffs, eps)
    rows, cols = np.shape(W)
    s = shape_scale(rows, cols, scale_mode)
    return dict(W=apply_update(W, O, lr, weight_decay, s), M=M_new, O=O, nu=nu, finite=True)
