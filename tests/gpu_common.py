"""Shared helpers of the GPU parity tests (inputs, oracle replay, error measures)."""
from __future__ import annotations

import numpy as np

import oracle
from synthetic import round_bf16

BF16_TOL = 2e-2   # relative Frobenius error per matrix, bf16 path
F32_TOL = 1e-4    # relative Frobenius error per matrix, fp32 path

# The update O read back through a bf16 weight.  With W = 0 the step stores
# W_after = RNE_bf16(-lr s O_gpu).  bf16 carries an 8-bit significand, so round to
# nearest even moves every element by at most 2^-8 of its magnitude:
# ||RNE(x) - x|| <= 2^-8 ||x||.  Hence, for O_read = -W_after / (lr s),
#   rel_f(O_read, O_ref) <= rel_f(O_gpu, O_ref) + 2^-8 (1 + rel_f(O_gpu, O_ref)),
# and the 2e-2 bound on O_gpu becomes this bound on what the test can read.
BF16_UPDATE_TOL = BF16_TOL + 2.0 ** -8 * (1.0 + BF16_TOL)


def torch_mod():
    import torch
    return torch


def to_device(a: np.ndarray, dtype: str):
    """Exact upload: `a` holds values representable in `dtype` (bf16-rounded or float32)."""
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda().contiguous()


def to_numpy(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_f(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at each value of x (the largest RNE rounding error)."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 1e-38)))
    return 0.5 * np.exp2(e - 7)


def dominant_subspace_error(O_gpu, O_ref, U_in, thresh=1e-2) -> float:
    """Error of O restricted to the left singular directions of the input whose
    normalised singular value is >= thresh (wide orientation handled)."""
    X = np.asarray(U_in, np.float64)
    t = X.shape[0] > X.shape[1]
    if t:
        X, O_gpu, O_ref = X.T, np.asarray(O_gpu).T, np.asarray(O_ref).T
    u, s, _ = np.linalg.svd(X / np.linalg.norm(X), full_matrices=False)
    P = u[:, s >= thresh]
    return rel_f(P.T @ O_gpu, P.T @ O_ref)


def oracle_step_sequence(W0, Gs, coeffs, **hp):
    """Replay several oracle steps from M = 0; returns (W, M, last O, last nu)."""
    W = np.asarray(W0, np.float64)
    M = np.zeros_like(W)
    r = None
    for G in Gs:
        r = oracle.muon_step(W, G, M, coeffs, **hp)
        W, M = r["W"], r["M"]
    return W, M, r["O"], r["nu"]


def bf16_values(a) -> np.ndarray:
    return round_bf16(np.asarray(a, np.float32))


def update_from_zero_weights(W_after, lr, s) -> np.ndarray:
    """O recovered from a step taken with W = 0: W_after = -lr s O (rounded to W's dtype)."""
    return -to_numpy(W_after) / (lr * s)
