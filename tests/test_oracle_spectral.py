"""Pins of the power iteration and the spectral cap (no GPU)."""
import numpy as np

import oracle
from synthetic import gaussian, gaussian_spike, rng_for


def _with_spectrum(m, n, s, seed):
    rng = rng_for(seed, 0)
    U, _ = np.linalg.qr(rng.standard_normal((m, len(s))))
    V, _ = np.linalg.qr(rng.standard_normal((n, len(s))))
    return (U * s) @ V.T, U, V


def test_power_iteration_converges_to_svd_with_a_gap():
    s = np.concatenate([[5.0, 2.0], np.linspace(1.5, 0.1, 30)])
    W, U, V = _with_spectrum(40, 70, s, 1)
    v0 = rng_for(2, 0).standard_normal(70)
    u, v, sigma = oracle.power_iteration(W, v0, 30)
    assert abs(sigma - 5.0) < 1e-12
    assert abs(abs(u @ U[:, 0]) - 1) < 1e-12 and abs(abs(v @ V[:, 0]) - 1) < 1e-12
    # ratio (2/5)^2 per step: 3 steps leave a relative error near 0.4^6 in sigma
    _, _, s3 = oracle.power_iteration(W, v0, 3)
    assert s3 <= 5.0 and s3 > 5.0 * (1 - 0.05)


def test_power_iteration_matches_lapack_on_spike_gradient():
    G = gaussian_spike(rng_for(1000, 3), 300, 120, rank=1)  # a distinct top singular value
    u, v, sigma = oracle.power_iteration(G, np.ones(120), 50)
    assert abs(sigma - np.linalg.svd(G, compute_uv=False)[0]) / sigma < 1e-6


def test_stable_rank_limits():
    Q, _ = np.linalg.qr(gaussian(rng_for(3, 0), 60, 20))
    assert abs(oracle.stable_rank(Q.T, 1.0) - 20) < 1e-12
    r1 = np.outer(np.arange(1, 5.0), np.arange(1, 8.0))
    assert abs(oracle.stable_rank(r1, np.linalg.norm(r1, 2)) - 1) < 1e-12


def test_cap_removes_first_order_growth_of_sigma_max():
    s = np.concatenate([[3.0, 1.0], np.linspace(0.9, 0.05, 20)])
    W, U, V = _with_spectrum(30, 50, s, 4)
    u, v = U[:, 0], V[:, 0]
    O = gaussian(rng_for(5, 0), 30, 50) + 2.0 * np.outer(u, v)
    Oc, alpha = oracle.spectral_cap(O, u, v)
    assert abs(u @ Oc @ v) < 1e-12 and abs(alpha - u @ O @ v) < 1e-12
    # second-order term of sigma_max(W + E) is at most ||E||^2 / (sigma_1 - sigma_2)
    K = 2 * np.linalg.norm(O, 2) ** 2 / (3.0 - 1.0)
    for eta in (1e-3, 1e-4):
        grow_c = np.linalg.norm(W + eta * Oc, 2) - 3.0
        grow_u = np.linalg.norm(W + eta * O, 2) - 3.0
        assert abs(eta * alpha) > 20 * K * eta ** 2             # the first-order term dominates here
        assert abs(grow_u - eta * alpha) < K * eta ** 2         # uncapped: grows at first order
        assert abs(grow_c) < K * eta ** 2                       # capped: second order only
    # everything orthogonal to u (or to v) passes unchanged
    P = np.eye(30) - np.outer(u, u)
    assert np.allclose(P @ Oc, P @ O, atol=1e-13)


def test_capped_step_matches_plain_step_when_direction_is_orthogonal():
    rng = rng_for(6, 0)
    W = rng.standard_normal((20, 30)) * 0.02
    G = rng.standard_normal((20, 30))
    q5 = [oracle.QUINTIC] * 5
    plain = oracle.muon_step(W, G, np.zeros_like(G), q5)
    u = np.zeros(20)
    v = np.zeros(30)
    capped = oracle.muon_step_capped(W, G, np.zeros_like(G), q5, u, v)
    assert np.allclose(capped["W"], plain["W"], rtol=0, atol=1e-15) and capped["alpha"] == 0.0


def test_min_singular_reaches_lapack_with_a_bottom_gap():
    s = np.concatenate([np.linspace(3.0, 1.0, 29), [0.1]])  # full rank: 30 singular values
    for m, n in ((30, 50), (50, 30)):  # wide and tall: the iteration runs on the short side
        W, U, V = _with_spectrum(m, n, s, 3)
        y0 = rng_for(4, 0).standard_normal(min(m, n))
        y, smin = oracle.min_singular_shifted(W, y0, 3.0, 300)
        # rate (9 - 1) / (9 - 0.01) per step on y; the Rayleigh value converges at its square
        assert abs(smin - 0.1) < 1e-9
        bottom = U[:, -1] if m <= n else V[:, -1]
        assert abs(abs(y @ bottom) - 1) < 1e-9


def test_min_singular_is_exact_on_semi_orthogonal_and_an_upper_bound_otherwise():
    Q, _ = np.linalg.qr(rng_for(5, 0).standard_normal((90, 40)))
    _, smin = oracle.min_singular_shifted(Q.T, np.ones(40), 1.0, 3)
    assert abs(smin - 1.0) < 1e-13
    G = gaussian(rng_for(6, 0), 40, 70)
    true_min = np.linalg.svd(G, compute_uv=False)[-1]
    for k in (0, 1, 5, 40):
        _, est = oracle.min_singular_shifted(G, np.ones(40), np.linalg.norm(G, 2), k)
        assert est >= true_min * (1 - 1e-12)


def test_min_singular_brute_force_two_by_three():
    # W W^T = diag(4, 1): sigma = (2, 1); one shifted step from (1, 1) with s = 4 gives y = (0, 3) / 3
    W = np.array([[2.0, 0.0, 0.0], [0.0, 0.6, 0.8]])
    y, smin = oracle.min_singular_shifted(W, np.array([1.0, 1.0]), 2.0, 1)
    assert np.allclose(y, [0.0, 1.0], rtol=0, atol=1e-15)
    assert abs(smin - 1.0) < 1e-15
