"""Pins of the fp64 oracle to facts other than itself (no GPU).

Each test is chosen so that a plausible slip in the oracle -- a dropped
polynomial term, a sign, XX^T vs X^T X, B X vs X B, a missing transpose back,
the wrong Nesterov buffer, weight decay applied after the step -- fails it.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from synthetic import gaussian, gaussian_spike, ill_conditioned, rng_for
from tests.nsref import f_k, f_k_exact, polar_factor, rel_f, svd_closed_form

QUINTIC5 = [oracle.QUINTIC] * 5
CUBIC10 = [oracle.CUBIC] * 10


# ---- T1: SVD closed form of the iteration --------------------------------
@pytest.mark.parametrize("shape", [(16, 40), (40, 16), (33, 33), (7, 129)])
@pytest.mark.parametrize("coeffs", [CUBIC10, QUINTIC5, [(2.0, -1.5, 0.5), (1.7, -0.9, 0.2), oracle.CUBIC]])
def test_closed_form_matches_svd(shape, coeffs):
    rng = rng_for(11, shape[0] * 1000 + shape[1])
    G = gaussian(rng, *shape)
    O, nu = oracle.orthogonalize(G, coeffs, eps=0.0)
    expect = svd_closed_form(G / np.linalg.norm(G), coeffs)
    assert rel_f(O, expect) <= 1e-12
    assert O.shape == G.shape


# ---- T2: polar factor on the 128x64 cubic case ----------------------------
def test_polar_factor_cubic_128x64():
    G = gaussian(rng_for(0, 0), 128, 64).astype(np.float32).astype(np.float64)
    O, _ = oracle.orthogonalize(G, CUBIC10, eps=1e-7)
    assert rel_f(O, svd_closed_form(G / (np.linalg.norm(G) + 1e-7), CUBIC10)) <= 1e-12
    # 10 cubic steps from normalised singular values in [0.04, 0.21] land within 2e-3 of U V^T
    assert rel_f(O, polar_factor(G)) < 2e-3
    O20, _ = oracle.orthogonalize(G, [oracle.CUBIC] * 20, eps=1e-7)
    assert rel_f(O20, polar_factor(G)) < 1e-10


# ---- T3: semi-orthogonal inputs are scaled, not turned ----------------------
@pytest.mark.parametrize("m,n", [(64, 128), (96, 96), (48, 200)])
@pytest.mark.parametrize("coeffs", [CUBIC10, QUINTIC5])
def test_semi_orthogonal_fixed_direction(m, n, coeffs):
    q, _ = np.linalg.qr(gaussian(rng_for(5, m), n, m))
    Q = q.T  # m x n, rows orthonormal
    O, nu = oracle.orthogonalize(Q, coeffs, eps=0.0)
    assert abs(nu - np.sqrt(m)) < 1e-12
    assert rel_f(O, f_k(1.0 / np.sqrt(m), coeffs) * Q) <= 1e-12
    if coeffs is CUBIC10 and m == 64:
        assert abs(f_k(1.0 / np.sqrt(m), coeffs) - 1.0) < 1e-9


# ---- T4: output singular values lie in the polynomial's band -------------
def test_quintic_band_on_spike_gradient():
    # out_proj shape (768 x 1536), Gaussian bulk + rank-4 spike
    G = gaussian_spike(rng_for(1000, 0), 768, 1536)
    O, _ = oracle.orthogonalize(G, QUINTIC5)
    s_out = np.linalg.svd(O, compute_uv=False)
    s_in = np.linalg.svd(G / np.linalg.norm(G), compute_uv=False)
    grid = np.linspace(1e-6, 1.0, 400001)
    fg = f_k(grid, QUINTIC5)
    assert abs(fg.max() - 1.2024) < 1e-3  # sup of f_5 over (0, 1]
    inside = (grid >= s_in.min()) & (grid <= s_in.max())
    lo, hi = fg[inside].min(), fg[inside].max()
    assert s_out.max() <= fg.max() + 1e-9
    assert lo - 1e-6 <= s_out.min() and s_out.max() <= hi + 1e-6
    if s_in.min() >= 1e-2:
        assert s_out.min() >= 0.6817 and s_out.max() <= 1.1345


def test_band_lower_edge_matches_scalar():
    G = ill_conditioned(rng_for(3000, 1), 64, 96)
    O, _ = oracle.orthogonalize(G, QUINTIC5, eps=0.0)
    s_in = np.linalg.svd(G / np.linalg.norm(G), compute_uv=False)
    s_out = np.sort(np.linalg.svd(O, compute_uv=False))
    expect = np.sort([f_k(float(s), QUINTIC5) for s in s_in])
    assert np.allclose(s_out, expect, rtol=1e-8, atol=1e-12)


# ---- exact rational arithmetic on inputs with rational SVDs ----------------
def _rot(p, q, r):  # rational rotation from a Pythagorean triple p^2+q^2=r^2
    return [[Fraction(p, r), Fraction(-q, r)], [Fraction(q, r), Fraction(p, r)]]


@pytest.mark.parametrize("coeffs", [[oracle.CUBIC] * 3, [oracle.QUINTIC] * 2])
def test_exact_fractions_rotated_diagonal(coeffs):
    # X = R1 diag(3, 4) [I 0] R2^T  with R1, R2 rational rotations, ||X||_F = 5.
    R1 = _rot(3, 4, 5)
    R2 = [[Fraction(5, 13), Fraction(-12, 13), 0], [Fraction(12, 13), Fraction(5, 13), 0], [0, 0, 1]]
    D = [[Fraction(3), 0, 0], [0, Fraction(4), 0]]
    mul = lambda P, Q: [[sum(P[i][t] * Q[t][j] for t in range(len(Q))) for j in range(len(Q[0]))] for i in range(len(P))]
    tr = lambda P: [list(r) for r in zip(*P)]
    X = mul(mul(R1, D), tr(R2))
    fD = [[f_k_exact(Fraction(3, 5), coeffs), 0, 0], [0, f_k_exact(Fraction(4, 5), coeffs), 0]]
    expect = np.array(mul(mul(R1, fD), tr(R2)), dtype=np.float64)
    got, nu = oracle.orthogonalize(np.array(X, dtype=np.float64), coeffs, eps=0.0)
    assert abs(nu - 5.0) < 1e-14
    assert np.max(np.abs(got - expect)) < 1e-13
    gotT, _ = oracle.orthogonalize(np.array(X, dtype=np.float64).T, coeffs, eps=0.0)
    assert np.max(np.abs(gotT - expect.T)) < 1e-13


# ---- T5: invariances --------------------------------------------------------
def test_invariances():
    G = gaussian(rng_for(7, 1), 24, 40)
    O, _ = oracle.orthogonalize(G, QUINTIC5, eps=0.0)
    O2, _ = oracle.orthogonalize(37.5 * G, QUINTIC5, eps=0.0)
    assert rel_f(O2, O) < 1e-13
    OT, _ = oracle.orthogonalize(G.T, QUINTIC5, eps=0.0)
    assert rel_f(OT, O.T) < 1e-13
    P, _ = np.linalg.qr(gaussian(rng_for(7, 2), 24, 24))
    Q, _ = np.linalg.qr(gaussian(rng_for(7, 3), 40, 40))
    Opq, _ = oracle.orthogonalize(P @ G @ Q, QUINTIC5, eps=0.0)
    assert rel_f(Opq, P @ O @ Q) < 1e-12


def test_first_step_independent_of_beta_and_convention():
    rng = rng_for(8, 0)
    W = rng.standard_normal((20, 30)) * 0.02
    G = rng.standard_normal((20, 30))
    Z = np.zeros_like(G)
    r1 = oracle.muon_step(W, G, Z, QUINTIC5, beta=0.95, eps=0.0)
    r2 = oracle.muon_step(W, G, Z, QUINTIC5, beta=0.5, eps=0.0)
    assert rel_f(r1["O"], r2["O"]) < 1e-13
    # EMA convention: M <- beta M + (1-beta) G ; U = (1-beta) G + beta M  ==  (1-beta) * SGD-form U
    beta = 0.9
    G2 = rng.standard_normal((20, 30))
    M_sgd = oracle.momentum_update(Z, G, beta)
    M_sgd = oracle.momentum_update(M_sgd, G2, beta)
    U_sgd = oracle.nesterov_lookahead(G2, M_sgd, beta)
    M_ema = (1 - beta) * G
    M_ema = beta * M_ema + (1 - beta) * G2
    U_ema = (1 - beta) * G2 + beta * M_ema
    O_sgd, _ = oracle.orthogonalize(U_sgd, QUINTIC5, eps=0.0)
    O_ema, _ = oracle.orthogonalize(U_ema, QUINTIC5, eps=0.0)
    assert rel_f(O_sgd, O_ema) < 1e-12


# ---- momentum, Nesterov, decay: closed forms over several steps -------------
def test_momentum_closed_form_and_nesterov():
    rng = rng_for(9, 0)
    beta = 0.95
    Gs = [rng.standard_normal((6, 9)) for _ in range(7)]
    M = np.zeros((6, 9))
    for t, G in enumerate(Gs):
        M = oracle.momentum_update(M, G, beta)
        closed = sum(beta ** (t - j) * Gs[j] for j in range(t + 1))
        assert np.allclose(M, closed, rtol=1e-14, atol=1e-14)
        U = oracle.nesterov_lookahead(G, M, beta)
        assert np.allclose(U, G + beta * closed, rtol=1e-14, atol=1e-14)


def test_step_decay_and_scale():
    rng = rng_for(9, 1)
    W = rng.standard_normal((30, 10))
    Z = np.zeros((30, 10))
    r = oracle.muon_step(W, Z, Z, QUINTIC5, lr=0.02, weight_decay=0.1)
    assert r["finite"] and np.all(r["O"] == 0)
    assert np.array_equal(r["W"], W * (1 - 0.02 * 0.1))
    G = rng.standard_normal((30, 10))
    r = oracle.muon_step(W, G, Z, QUINTIC5, lr=0.5, weight_decay=0.0, eps=0.0, nesterov=False)
    O, _ = oracle.orthogonalize(G, QUINTIC5, eps=0.0)
    assert np.allclose(r["W"], W - 0.5 * np.sqrt(3.0) * O, rtol=0, atol=1e-14)
    assert oracle.shape_scale(768, 1536) == 1.0
    assert abs(oracle.shape_scale(3352, 768) - 2.08916) < 1e-5
    assert abs(oracle.shape_scale(8768, 2048) - 2.0691) < 1e-4
    assert oracle.shape_scale(3352, 768, oracle.SCALE_NONE) == 1.0
    assert abs(oracle.shape_scale(3352, 768, oracle.SCALE_RMS_MATCH) - 0.2 * np.sqrt(3352)) < 1e-12


def test_nonfinite_policy():
    W = np.ones((4, 6))
    G = np.ones((4, 6))
    G[1, 2] = np.inf
    r = oracle.muon_step(W, G, np.zeros_like(G), QUINTIC5)
    assert not r["finite"] and np.array_equal(r["W"], W)


def test_golden_fixture_regression():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.txt")
    cases = {}
    with open(path) as f:
        name = None
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case "):
                name = line.split()[1]
                cases[name] = []
            else:
                cases[name].append([float(v) for v in line.split()])
    G = gaussian(rng_for(42, 0), 5, 3)
    O, _ = oracle.orthogonalize(G, CUBIC10)
    assert np.allclose(O, np.array(cases["cubic10_5x3"]), rtol=0, atol=1e-15)
    O, _ = oracle.orthogonalize(G.T, QUINTIC5)
    assert np.allclose(O, np.array(cases["quintic5_3x5"]), rtol=0, atol=1e-15)


def _loops_step(W, G, M, coeffs, lr, beta, wd, eps, scale):
    """The whole step with explicit Python loops over scalars (no NumPy arithmetic)."""
    R, C = len(W), len(W[0])
    Mn = [[beta * M[i][j] + G[i][j] for j in range(C)] for i in range(R)]
    U = [[G[i][j] + beta * Mn[i][j] for j in range(C)] for i in range(R)]
    nu = sum(U[i][j] ** 2 for i in range(R) for j in range(C)) ** 0.5
    X = [[U[i][j] / (nu + eps) for j in range(C)] for i in range(R)]
    tall = R > C
    if tall:
        X = [[X[i][j] for i in range(R)] for j in range(C)]
    m, n = len(X), len(X[0])
    for a, b, c in coeffs:
        A = [[sum(X[i][k] * X[j][k] for k in range(n)) for j in range(m)] for i in range(m)]
        AA = [[sum(A[i][k] * A[k][j] for k in range(m)) for j in range(m)] for i in range(m)]
        B = [[b * A[i][j] + c * AA[i][j] for j in range(m)] for i in range(m)]
        X = [[a * X[i][j] + sum(B[i][k] * X[k][j] for k in range(m)) for j in range(n)] for i in range(m)]
    O = [[X[j][i] for j in range(m)] for i in range(n)] if tall else X
    Wn = [[W[i][j] * (1 - lr * wd) - lr * scale * O[i][j] for j in range(C)] for i in range(R)]
    return Wn, Mn


@pytest.mark.parametrize("shape", [(2, 3), (3, 5), (5, 3)])
def test_brute_force_loops_tiny(shape):
    """T6: the oracle's step equals a scalar-loop transcription of the definitions on tiny inputs."""
    R, C = shape
    rng = rng_for(77, R * 10 + C)
    W = rng.standard_normal(shape) * 0.02
    G = rng.standard_normal(shape)
    M = rng.standard_normal(shape) * 0.1
    coeffs = [oracle.QUINTIC] * 3 + [oracle.CUBIC] * 2
    s = oracle.shape_scale(R, C, oracle.SCALE_SQRT_RATIO)
    r = oracle.muon_step(W, G, M, coeffs, lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7)
    Wl, Ml = _loops_step(W.tolist(), G.tolist(), M.tolist(), coeffs, 0.02, 0.95, 0.1, 1e-7, s)
    assert np.allclose(r["W"], np.array(Wl), rtol=0, atol=1e-13)
    assert np.allclose(r["M"], np.array(Ml), rtol=0, atol=1e-13)
