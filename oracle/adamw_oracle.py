"""Plain float64 AdamW for the parameters Muon does not take -- TEST INFRASTRUCTURE ONLY.

Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
Muon is compared with AdamW on Mamba-2 130M under a protocol that varies
only which weight groups (input projection, output projection, both) are
trained with Muon; every other parameter -- and the projections Muon does
not take -- is trained with AdamW.  The practitioner notes (Muon Meets
Mamba blog, section 3.3) split the parameters by name into a spectral group
and a normal group.

READING: the pages name AdamW but not its form; this is the standard one
with bias correction and decoupled decay taken from the pre-step weights:
    m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
    W <- W (1 - lr wd) - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
"""
from __future__ import annotations

import numpy as np


def adamw_step(W, G, m, v, step, lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1):
    """One AdamW step (t = step >= 1).  Returns (W, m, v) as new float64 arrays."""
    W = np.asarray(W, np.float64)
    G = np.asarray(G, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * G
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * G * G
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    W = W * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return W, m, v


def select_muon(name: str, shape, mode: str = "both") -> bool:
    """Which parameters Muon takes: 2-D projection weights chosen by name.

    mode 'out_proj' / 'in_proj' / 'both' follows the protocol of the Muon
    Meets Mamba abstract; anything else (embeddings, norms, convolutions,
    A_log, D, dt biases, 1-D tensors) goes to AdamW.
    """
    if len(shape) != 2:
        return False
    if mode == "both":
        return "in_proj" in name or "out_proj" in name
    return mode in name
