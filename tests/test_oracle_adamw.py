"""Pins of the fp64 AdamW oracle and the parameter selection (no GPU)."""
import numpy as np

import oracle
from synthetic import rng_for


def test_first_step_is_signed_lr():
    # t = 1: m_hat = g and v_hat = g^2, so the step is lr * g / (|g| + eps)
    rng = rng_for(51, 0)
    W = rng.standard_normal((7, 9))
    G = rng.standard_normal((7, 9))
    Wn, m, v = oracle.adamw_step(W, G, np.zeros_like(W), np.zeros_like(W), 1, lr=0.01, eps=1e-8, weight_decay=0.0)
    assert np.allclose(W - Wn, 0.01 * G / (np.abs(G) + 1e-8), rtol=1e-12, atol=1e-15)
    assert np.allclose(m, 0.1 * G) and np.allclose(v, 0.05 * G * G)


def test_moment_closed_forms_over_steps():
    rng = rng_for(51, 1)
    b1, b2 = 0.9, 0.95
    Gs = [rng.standard_normal((4, 5)) for _ in range(6)]
    W = rng.standard_normal((4, 5))
    m = np.zeros_like(W)
    v = np.zeros_like(W)
    for t, G in enumerate(Gs, start=1):
        W, m, v = oracle.adamw_step(W, G, m, v, t, beta1=b1, beta2=b2)
        m_cf = sum((1 - b1) * b1 ** (t - j) * Gs[j - 1] for j in range(1, t + 1))
        v_cf = sum((1 - b2) * b2 ** (t - j) * Gs[j - 1] ** 2 for j in range(1, t + 1))
        assert np.allclose(m, m_cf, rtol=1e-13) and np.allclose(v, v_cf, rtol=1e-13)
        # constant gradient: bias-corrected moments equal g and g^2 exactly
    Wc = np.ones((2, 2))
    m = np.zeros((2, 2))
    v = np.zeros((2, 2))
    g = np.full((2, 2), 0.3)
    for t in range(1, 5):
        W1, m, v = oracle.adamw_step(Wc, g, m, v, t, lr=1.0, eps=0.0, weight_decay=0.0)
        assert np.allclose(Wc - W1, 1.0, rtol=1e-12)


def test_decay_only_and_scale_invariance():
    W = np.full((3, 3), 2.0)
    Z = np.zeros((3, 3))
    Wn, _, _ = oracle.adamw_step(W, Z, Z, Z, 1, lr=0.1, weight_decay=0.5)
    assert np.array_equal(Wn, W * (1 - 0.05))
    rng = rng_for(51, 2)
    G = rng.standard_normal((3, 3))
    a, _, _ = oracle.adamw_step(W, G, Z, Z, 3, eps=0.0)
    b, _, _ = oracle.adamw_step(W, 1e4 * G, Z, Z, 3, eps=0.0)
    assert np.allclose(a, b, rtol=1e-12)


def test_selection_by_name_and_shape():
    assert oracle.select_muon("layers.0.mixer.in_proj.weight", (3352, 768), "both")
    assert oracle.select_muon("layers.0.mixer.out_proj.weight", (768, 1536), "out_proj")
    assert not oracle.select_muon("layers.0.mixer.in_proj.weight", (3352, 768), "out_proj")
    assert not oracle.select_muon("layers.0.mixer.D", (24,), "both")
    assert not oracle.select_muon("embeddings.weight", (50280, 768), "both")
    assert not oracle.select_muon("layers.0.mixer.conv1d.weight", (1792, 1, 4), "both")
