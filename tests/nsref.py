"""Helpers for pins that do not go through the oracle's matrix iteration.

Scalar polynomial composition f_k(s) = p_k(...p_1(s)) with p(s) = a s + b s^3 + c s^5
(evaluated in plain Python floats or exact Fractions), and the SVD closed form
U f_k(S) V^T of k Newton-Schulz steps.
"""
from fractions import Fraction

import numpy as np


def f_k(s, coeffs):
    for (a, b, c) in coeffs:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def f_k_exact(s: Fraction, coeffs):
    fc = [(Fraction(str(a)), Fraction(str(b)), Fraction(str(c))) for (a, b, c) in coeffs]
    for (a, b, c) in fc:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def svd_closed_form(X0, coeffs):
    """U f_k(S) V^T for X0 = U S V^T, using LAPACK's SVD and the scalar polynomial."""
    U, S, Vt = np.linalg.svd(np.asarray(X0, np.float64), full_matrices=False)
    fS = np.array([f_k(float(s), coeffs) for s in S])
    return (U * fS) @ Vt


def polar_factor(X):
    U, _, Vt = np.linalg.svd(np.asarray(X, np.float64), full_matrices=False)
    return U @ Vt


def rel_f(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
