"""Plant plausible mistakes in copies of the oracle's iteration (CPU only) and
check that the closed-form pin rejects every one of them."""
import numpy as np
import pytest

import oracle
from synthetic import gaussian, rng_for
from tests.nsref import rel_f, svd_closed_form


def _ns_dropped_c(X, coeffs):
    for a, b, c in coeffs:
        A = X @ X.T
        X = a * X + (b * A) @ X
    return X


def _ns_wrong_sign(X, coeffs):
    for a, b, c in coeffs:
        A = X @ X.T
        X = a * X - (b * A + c * A @ A) @ X
    return X


def _ns_gram_transposed(X, coeffs):  # A = X^T X on a square input
    for a, b, c in coeffs:
        A = X.T @ X
        X = a * X + (b * A + c * A @ A) @ X
    return X


def _ns_right_multiply(X, coeffs):  # X B instead of B X (square input)
    for a, b, c in coeffs:
        A = X @ X.T
        X = a * X + X @ (b * A + c * A @ A)
    return X


def _ns_coeffs_reversed(X, coeffs):  # iterates coefficient triples in the wrong order
    return oracle.newton_schulz(X, list(reversed(coeffs)))


MUTANTS = [_ns_dropped_c, _ns_wrong_sign, _ns_gram_transposed, _ns_right_multiply, _ns_coeffs_reversed]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_closed_form_pin_rejects(mutant):
    G = gaussian(rng_for(77, 0), 24, 24)  # square, so shape errors cannot hide a mistake
    G = G + 0.3 * np.eye(24)  # non-normal, non-symmetric
    X0 = G / np.linalg.norm(G)
    coeffs = [oracle.QUINTIC, (2.0, -1.5, 0.5), oracle.CUBIC]
    good = oracle.newton_schulz(X0, coeffs)
    bad = mutant(X0, coeffs)
    ref = svd_closed_form(X0, coeffs)
    assert rel_f(good, ref) < 1e-12
    assert rel_f(bad, ref) > 1e-6


def test_missing_transpose_back_rejected():
    G = gaussian(rng_for(77, 1), 40, 16)
    O, _ = oracle.orthogonalize(G, [oracle.QUINTIC] * 5, eps=0.0)
    ref = svd_closed_form(G / np.linalg.norm(G), [oracle.QUINTIC] * 5)
    assert O.shape == ref.shape and rel_f(O, ref) < 1e-12
    wrong = oracle.newton_schulz((G / np.linalg.norm(G)).T, [oracle.QUINTIC] * 5)  # left wide
    assert wrong.shape != ref.shape
