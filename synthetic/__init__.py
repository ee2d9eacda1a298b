"""Seeded synthetic inputs shared by the oracle-side tests, the CUDA-side tests and bench.py.

This module draws random numbers and rounds them to the storage formats the
optimizer consumes.  It holds none of the optimizer's arithmetic (no momentum,
normalisation, Newton-Schulz or update rule), so both the oracle and the CUDA
path may import it without sharing any of the method.

Workload shapes follow a Mamba-2 130M model (d_model 768, d_inner 1536,
d_state 128, one group, 24 heads, 24 layers): the output projection is
768 x 1536 (PyTorch out x in) and the input projection is
(2*1536 + 2*128 + 24) x 768 = 3352 x 768.  The pages (Muon Meets Mamba:
Spectral Optimization for State Space Models, abstract) train exactly these
two weight groups but print no gradients, so the gradients are synthetic:
Gaussian noise plus a rank-4 spike, or a log-uniform spectrum for the
ill-conditioned variant.
"""
from __future__ import annotations

import numpy as np

# Mamba-2 130M projection shapes (rows, cols) in PyTorch (out, in) order.
MAMBA2_130M_OUT_PROJ = (768, 1536)
MAMBA2_130M_IN_PROJ = (3352, 768)
MAMBA2_130M_LAYERS = 24
# The other parameters of Mamba-2 130M (vocab 50280, conv width 4, 24 heads):
# the embedding (tied with the output head), per layer the depthwise conv
# weight and bias over d_inner + 2 d_state channels, A_log, D, dt_bias, the
# gated norm over d_inner and the block norm; the final norm.
def mamba2_130m_other_params():
    shapes = [("embeddings.weight", (50280, 768))]
    for layer in range(MAMBA2_130M_LAYERS):
        pre = f"layers.{layer}."
        shapes += [(pre + "mixer.conv1d.weight", (1792, 1, 4)), (pre + "mixer.conv1d.bias", (1792,)),
                   (pre + "mixer.A_log", (24,)), (pre + "mixer.D", (24,)), (pre + "mixer.dt_bias", (24,)),
                   (pre + "mixer.norm.weight", (1536,)), (pre + "norm.weight", (768,))]
    shapes.append(("norm_f.weight", (768,)))
    return shapes


# Scaled Mamba-2-style model: d_model 2048, d_inner 4096, 48 layers.
SCALED_2K_IN_PROJ = (8192 + 512 + 64, 2048)
SCALED_2K_OUT_PROJ = (2048, 4096)
SCALED_2K_LAYERS = 48


# --------------------------------------------------------------------------
# bf16 storage (round to nearest even), as a bit pattern and as its value.
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even) and return the uint16 bits.

    NaN stays NaN (quiet bit forced), infinities stay infinite.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    b = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = ((b[nan] >> 16) | 0x40).astype(np.uint16)
    return out


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Exact float32 value of bfloat16 bit patterns."""
    bits = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (bits.astype(np.uint32) << 16).view(np.float32)


def round_bf16(x) -> np.ndarray:
    """float32 values that are exactly representable in bfloat16 (RNE of x)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# --------------------------------------------------------------------------
# Seeds: seed = 1000*config + 10*step + group, matrix l uses default_rng([seed, l]).
# --------------------------------------------------------------------------
def seed_for(config: int, step: int, group: int) -> int:
    return 1000 * config + 10 * step + group


def rng_for(seed: int, index: int) -> np.random.Generator:
    return np.random.default_rng([seed, index])


def _orthonormal_columns(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))  # sign-fixed (Haar)


def gaussian_spike(rng: np.random.Generator, rows: int, cols: int, std: float = 1e-3,
                   rank: int = 4, factor: float = 10.0) -> np.ndarray:
    """Gaussian N(0, std^2) bulk plus a rank-`rank` spike (float64).

    The bulk's largest singular value is about std*(sqrt(rows)+sqrt(cols)); the
    spike's singular values are `factor` times that edge.
    """
    g = rng.standard_normal((rows, cols)) * std
    if rank > 0:
        u = _orthonormal_columns(rng, rows, rank)
        v = _orthonormal_columns(rng, cols, rank)
        sigma = factor * std * (np.sqrt(rows) + np.sqrt(cols))
        g += sigma * (u @ v.T)
    return g


def ill_conditioned(rng: np.random.Generator, rows: int, cols: int,
                    log10_lo: float = -6.0, log10_hi: float = 0.0) -> np.ndarray:
    """Q1 diag(s) Q2^T with Haar Q1, Q2 and s_i = 10**U(lo, hi) (condition ~1e6)."""
    k = min(rows, cols)
    q1 = _orthonormal_columns(rng, rows, k)
    q2 = _orthonormal_columns(rng, cols, k)
    s = 10.0 ** rng.uniform(log10_lo, log10_hi, size=k)
    return (q1 * s) @ q2.T


def gaussian(rng: np.random.Generator, rows: int, cols: int, std: float = 1.0) -> np.ndarray:
    return rng.standard_normal((rows, cols)) * std


def weights(rng: np.random.Generator, rows: int, cols: int, std: float = 0.02) -> np.ndarray:
    """Initial weights N(0, std^2): the plainest init (the pages give none)."""
    return rng.standard_normal((rows, cols)) * std


def draw(kind: str, rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    if kind == "spike":
        return gaussian_spike(rng, rows, cols)
    if kind == "ill":
        return ill_conditioned(rng, rows, cols)
    if kind == "gauss":
        return gaussian(rng, rows, cols)
    raise ValueError(f"unknown gradient kind {kind!r}")


def group_inputs(config: int, step: int, group: int, count: int, rows: int, cols: int,
                 kind: str = "spike", dtype: str = "bf16"):
    """Gradients for `count` same-shape matrices of one group at one step.

    Returns float32 arrays whose values are exactly what the device receives:
    bf16-rounded for dtype 'bf16', float32-rounded for 'f32'.
    """
    seed = seed_for(config, step, group)
    out = []
    for l in range(count):
        g = draw(kind, rng_for(seed, l), rows, cols)
        g32 = g.astype(np.float32)
        out.append(round_bf16(g32) if dtype == "bf16" else g32)
    return out


def group_weights(config: int, group: int, count: int, rows: int, cols: int, dtype: str = "bf16"):
    """Initial weights of one group (seed shares the scheme, step slot 9)."""
    seed = seed_for(config, 9, group) + 500
    out = []
    for l in range(count):
        w = weights(rng_for(seed, l), rows, cols).astype(np.float32)
        out.append(round_bf16(w) if dtype == "bf16" else w)
    return out
