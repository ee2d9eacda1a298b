"""The input recipe: the drawn gradients have the spectra the workloads call for (no method arithmetic)."""
import numpy as np

from synthetic import (MAMBA2_130M_IN_PROJ, MAMBA2_130M_OUT_PROJ, f32_to_bf16_bits, bf16_bits_to_f32,
                       gaussian_spike, ill_conditioned, mamba2_130m_other_params, rng_for, round_bf16)


def test_rank4_spike_sits_at_ten_times_the_bulk_edge():
    for rows, cols in (MAMBA2_130M_OUT_PROJ, MAMBA2_130M_IN_PROJ):
        g = gaussian_spike(rng_for(11, 0), rows, cols)
        s = np.linalg.svd(g, compute_uv=False)
        edge = 1e-3 * (np.sqrt(rows) + np.sqrt(cols))
        assert np.allclose(s[:4], 10 * edge, rtol=0.02)      # the spike
        assert 0.9 * edge < s[4] < 1.1 * edge                # the bulk's top edge, std 1e-3


def test_ill_conditioned_spectrum_is_log_uniform_over_six_decades():
    g = ill_conditioned(rng_for(12, 0), 300, 200)
    s = np.linalg.svd(g, compute_uv=False)
    assert s.max() <= 1.0 and s.min() >= 1e-6
    logs = np.log10(s)
    assert logs.max() - logs.min() > 5.0
    # roughly uniform in log10: each decade holds about a sixth of the values
    counts, _ = np.histogram(logs, bins=6, range=(-6, 0))
    assert counts.min() > 0.5 * len(s) / 6


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e38, 1e-40], np.float32)
    r = round_bf16(x)
    assert r[0] == 1.0
    assert r[1] == 1.0                      # halfway: to even (mantissa ...0)
    assert r[2] == 1.0 + 2.0 ** -6          # halfway: to even upward
    assert r[3] == -2.5
    assert np.array_equal(bf16_bits_to_f32(f32_to_bf16_bits(r)), r)


def test_other_parameters_of_mamba2_130m():
    ps = mamba2_130m_other_params()
    total = sum(int(np.prod(s)) for _, s in ps)
    assert len(ps) == 170 and total == 38887872
    names = [n for n, _ in ps]
    assert any("embedding" in n for n in names)
    assert not any("in_proj" in n or "out_proj" in n for n in names)
