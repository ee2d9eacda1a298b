"""Numerical facts the fp32 path relies on (three bf16 planes, six plane products), checked in NumPy."""
import numpy as np

from synthetic import rng_for, round_bf16


def split3(x):
    hi = round_bf16(x)
    mid = round_bf16((x.astype(np.float64) - hi).astype(np.float32))
    lo = round_bf16((x.astype(np.float64) - hi - mid).astype(np.float32))
    return hi.astype(np.float64), mid.astype(np.float64), lo.astype(np.float64)


def test_three_bf16_planes_reconstruct_fp32():
    x = (rng_for(5, 0).standard_normal(200000) * np.exp2(rng_for(5, 1).integers(-20, 20, 200000))).astype(np.float32)
    hi, mid, lo = split3(x)
    err = np.abs(x.astype(np.float64) - (hi + mid + lo))
    # each plane rounds the remainder to 8 significant bits: the residual is below 2^-24 |x|
    assert np.all(err <= np.abs(x.astype(np.float64)) * 2.0 ** -24)


def test_six_plane_products_cover_the_fp32_product():
    rng = rng_for(6, 0)
    a = rng.standard_normal((64, 256)).astype(np.float32)
    b = rng.standard_normal((256, 48)).astype(np.float32)
    ah, am, al = split3(a)
    bh, bm, bl = split3(b)
    kept = ah @ bh + ah @ bm + am @ bh + am @ bm + ah @ bl + al @ bh
    exact = a.astype(np.float64) @ b.astype(np.float64)
    dropped = am @ bl + al @ bm + al @ bl
    scale = np.abs(a.astype(np.float64)) @ np.abs(b.astype(np.float64))
    assert np.all(np.abs(dropped) <= scale * 2.0 ** -23)
    assert np.max(np.abs(kept - exact) / scale) <= 2.0 ** -22
    # two planes would not do: their error is far above fp32's resolution (2^-24)
    two = ah @ bh + ah @ bm + am @ bh
    assert np.max(np.abs(two - exact) / scale) > 2.0 ** -21
