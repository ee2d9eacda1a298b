"""Power iteration and the spectral-capped step vs the fp64 oracle (needs a B200)."""
import numpy as np
import pytest

import oracle
from synthetic import MAMBA2_130M_IN_PROJ, gaussian_spike, rng_for, round_bf16, weights
from tests.gpu_common import BF16_TOL, F32_TOL, rel_f, to_device, to_numpy

pytestmark = pytest.mark.gpu

# wide, tall, ragged (scalar paths: cols % 8 != 0), one past the 48 KB shared-memory default, and
# the streaming one-pass kernel at 6 and 8 vectors per lane (the out_proj width and its 2048
# limit), with a last stage of fewer than eight rows, at its 64-block cap (one matrix of 4000
# rows) and over the full out_proj batch (twelve blocks per matrix)
SHAPES = [(96, 200, 3), (200, 96, 2), (77, 45, 2), (45, 77, 1), (64, 13000, 1), (768, 1536, 2), (300, 2048, 2),
          (77, 48, 2), (4000, 512, 1), (768, 1536, 24)]


def _spiked(rows, cols, batch, seed, dtype):
    Ws = []
    for l in range(batch):
        W = gaussian_spike(rng_for(seed, l), rows, cols, rank=1)
        Ws.append(round_bf16(W) if dtype == "bf16" else W.astype(np.float32))
    return Ws


def _power(muon, Ws, v0s, iters, dtype):
    import torch
    W = [to_device(w, dtype) for w in Ws]
    u = [torch.zeros(w.shape[0], dtype=torch.float32, device="cuda") for w in Ws]
    v = [torch.from_numpy(v0.astype(np.float32)).cuda() for v0 in v0s]
    sigma = torch.zeros(len(Ws), dtype=torch.float32, device="cuda")
    muon.power_iteration(W, u, v, sigma, iters=iters)
    torch.cuda.synchronize()
    return [to_numpy(x) for x in u], [to_numpy(x) for x in v], to_numpy(sigma)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,cols,batch", SHAPES)
def test_power_iteration_matches_oracle(rows, cols, batch, dtype):
    from spectral_optimizer_state_b200 import Muon
    Ws = _spiked(rows, cols, batch, 71, dtype)
    v0s = [rng_for(72, l).standard_normal(cols).astype(np.float32) for l in range(batch)]
    with Muon() as muon:
        u, v, sigma = _power(muon, Ws, v0s, 6, dtype)
    for l in range(batch):
        ru, rv, rs = oracle.power_iteration(Ws[l].astype(np.float64), v0s[l].astype(np.float64), 6)
        # fp32 accumulation over at most 13000 terms of one sign-mixed dot product
        assert abs(sigma[l] - rs) <= 1e-5 * rs
        assert rel_f(u[l], ru) <= 1e-4
        assert rel_f(v[l], rv) <= 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_power_iteration_in_two_calls_continues_from_v(dtype):
    """One iteration, then two calls of three: each call leaves v normalised and its per-matrix
    block counters at zero, so 3 + 3 iterations are the oracle's 6 from the same start."""
    from spectral_optimizer_state_b200 import Muon
    rows, cols, batch = 200, 256, 3
    Ws = _spiked(rows, cols, batch, 74, dtype)
    v0s = [rng_for(75, l).standard_normal(cols).astype(np.float32) for l in range(batch)]
    with Muon() as muon:
        u1, v1, s1 = _power(muon, Ws, v0s, 1, dtype)
        _, vh, _ = _power(muon, Ws, v0s, 3, dtype)
        u6, v6, s6 = _power(muon, Ws, vh, 3, dtype)
    for l in range(batch):
        W = Ws[l].astype(np.float64)
        ru, rv, rs = oracle.power_iteration(W, v0s[l].astype(np.float64), 1)
        assert abs(s1[l] - rs) <= 1e-5 * rs and rel_f(u1[l], ru) <= 1e-4 and rel_f(v1[l], rv) <= 1e-4
        ru, rv, rs = oracle.power_iteration(W, v0s[l].astype(np.float64), 6)
        assert abs(s6[l] - rs) <= 1e-5 * rs and rel_f(u6[l], ru) <= 1e-4 and rel_f(v6[l], rv) <= 1e-4


def test_power_iteration_one_launch_per_iteration_when_blocks_do_not_fit():
    """fp32 rows of 2048 columns leave one block per SM, so 200 matrices cannot all be resident
    at once: the iterations then run as one launch each (no block waits on another) and must
    give the same results as the oracle."""
    from spectral_optimizer_state_b200 import Muon
    rows, cols, batch = 16, 2048, 200
    Ws = _spiked(rows, cols, batch, 76, "f32")
    v0s = [rng_for(77, l).standard_normal(cols).astype(np.float32) for l in range(batch)]
    with Muon() as muon:
        u, v, sigma = _power(muon, Ws, v0s, 3, "f32")
    for l in (0, 99, 199):
        ru, rv, rs = oracle.power_iteration(Ws[l].astype(np.float64), v0s[l].astype(np.float64), 3)
        assert abs(sigma[l] - rs) <= 1e-5 * rs
        assert rel_f(u[l], ru) <= 1e-4
        assert rel_f(v[l], rv) <= 1e-4


def test_power_iteration_reaches_the_svd_on_full_size_in_proj():
    """in_proj shape of the 130M model: 24 matrices with a planted top direction, 30 iterations."""
    from spectral_optimizer_state_b200 import Muon
    rows, cols = MAMBA2_130M_IN_PROJ
    Ws = _spiked(rows, cols, 24, 73, "bf16")
    v0s = [np.ones(cols, np.float32) for _ in range(24)]
    with Muon() as muon:
        _, v, sigma = _power(muon, Ws, v0s, 30, "bf16")
    for l in (0, 11, 23):
        _, s, Vt = np.linalg.svd(Ws[l].astype(np.float64), full_matrices=False)
        assert abs(sigma[l] - s[0]) <= 1e-4 * s[0]
        assert abs(abs(v[l] @ Vt[0]) - 1.0) <= 1e-4


def test_power_iteration_zero_matrix_gives_zero_triplet():
    from spectral_optimizer_state_b200 import Muon
    Ws = [np.zeros((40, 72), np.float32)]
    with Muon() as muon:
        u, v, sigma = _power(muon, Ws, [np.ones(72, np.float32)], 3, "f32")
    ru, rv, rs = oracle.power_iteration(Ws[0], np.ones(72), 3)
    assert sigma[0] == rs == 0.0
    assert not u[0].any() and not v[0].any() and not ru.any() and not rv.any()


def _capped_case(rows, cols, batch, dtype, seed):
    W0 = [weights(rng_for(seed, l), rows, cols) for l in range(batch)]
    G = [gaussian_spike(rng_for(seed + 1, l), rows, cols, rank=4) for l in range(batch)]
    if dtype == "bf16":
        W0 = [round_bf16(w) for w in W0]
        G = [round_bf16(g) for g in G]
    else:
        W0 = [w.astype(np.float32) for w in W0]
        G = [g.astype(np.float32) for g in G]
    uv = [oracle.power_iteration(w.astype(np.float64), np.ones(cols), 20)[:2] for w in W0]
    return W0, G, uv


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,cols,batch", [(192, 320, 2), (320, 192, 3), (77, 45, 1), (256, 256, 1)])
def test_step_capped_matches_oracle(rows, cols, batch, dtype):
    import torch
    from spectral_optimizer_state_b200 import Muon
    W0, G, uv = _capped_case(rows, cols, batch, dtype, 81)
    hp = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True, scale_mode=0)
    W = [to_device(w, dtype) for w in W0]
    Gd = [to_device(g, dtype) for g in G]
    M = [torch.zeros((rows, cols), dtype=torch.float32, device="cuda") for _ in range(batch)]
    u = [torch.from_numpy(x.astype(np.float32)).cuda() for x, _ in uv]
    v = [torch.from_numpy(y.astype(np.float32)).cuda() for _, y in uv]
    alpha = torch.zeros(batch, dtype=torch.float32, device="cuda")
    with Muon() as muon:
        coeffs = muon.get_coeffs()
        muon.step_capped(W, Gd, M, u, v, alpha, **hp)
        torch.cuda.synchronize()
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    a = to_numpy(alpha)
    for l in range(batch):
        # u, v as the kernel saw them (fp32)
        ul, vl = uv[l][0].astype(np.float32).astype(np.float64), uv[l][1].astype(np.float32).astype(np.float64)
        r = oracle.muon_step_capped(W0[l].astype(np.float64), G[l].astype(np.float64), np.zeros((rows, cols)),
                                    coeffs, ul, vl, **hp)
        dW_ref = r["W"] - W0[l]
        dW = to_numpy(W[l]) - W0[l]
        if dtype == "f32":
            assert rel_f(dW, dW_ref) <= tol
        else:
            # the bf16 store of W rounds each element by at most half a bf16 ulp of the new value
            assert rel_f(dW, dW_ref) <= tol + np.linalg.norm(np.abs(r["W"]) * 2.0 ** -8) / np.linalg.norm(dW_ref)
        # |d alpha| = |u^T dO v| <= ||dO||_2 <= ||dO||_F
        O_norm = np.linalg.norm(r["O"] + r["alpha"] * np.outer(ul, vl))
        assert abs(a[l] - r["alpha"]) <= tol * O_norm
        assert rel_f(to_numpy(M[l]), r["M"]) <= 1e-6


def test_capped_update_has_no_component_along_the_top_pair():
    """fp32 W: u^T (W_new - decay W_old) v is zero up to the orthogonalisation error."""
    import torch
    from spectral_optimizer_state_b200 import Muon
    rows, cols = 320, 192
    W0, G, uv = _capped_case(rows, cols, 1, "f32", 91)
    W = [to_device(W0[0], "f32")]
    M = [torch.zeros((rows, cols), dtype=torch.float32, device="cuda")]
    u = [torch.from_numpy(uv[0][0].astype(np.float32)).cuda()]
    v = [torch.from_numpy(uv[0][1].astype(np.float32)).cuda()]
    alpha = torch.zeros(1, dtype=torch.float32, device="cuda")
    lr, wd = 0.02, 0.1
    with Muon() as muon:
        muon.step_capped(W, [to_device(G[0], "f32")], M, u, v, alpha, lr=lr, weight_decay=wd)
        torch.cuda.synchronize()
    dW = to_numpy(W[0]) - (1 - lr * wd) * W0[0].astype(np.float64)
    ul, vl = to_numpy(u[0]), to_numpy(v[0])
    assert abs(ul @ dW @ vl) <= 1e-5 * np.linalg.norm(dW)
    assert abs(to_numpy(alpha)[0]) > 1e-3  # the cap removed something


def test_step_capped_rejects_missing_vectors():
    import torch
    from spectral_optimizer_state_b200 import Muon, MuonError
    W = [torch.zeros((64, 64), dtype=torch.float32, device="cuda")]
    with Muon() as muon:
        with pytest.raises((MuonError, ValueError)):
            muon.step_capped(W, W, [w.clone() for w in W], [], [], torch.zeros(1, device="cuda"))


def _min_singular(muon, Ws, y0s, smax, iters, dtype):
    import torch
    W = [to_device(w, dtype) for w in Ws]
    y = [torch.from_numpy(y0.astype(np.float32)).cuda() for y0 in y0s]
    sm = torch.from_numpy(np.asarray(smax, np.float32)).cuda()
    out = torch.zeros(len(Ws), dtype=torch.float32, device="cuda")
    muon.min_singular(W, y, sm, out, iters=iters)
    torch.cuda.synchronize()
    return [to_numpy(t) for t in y], to_numpy(out)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,cols,batch", SHAPES)
@pytest.mark.parametrize("iters", [0, 20])
def test_min_singular_matches_oracle(rows, cols, batch, dtype, iters):
    from spectral_optimizer_state_b200 import Muon
    Ws = [weights(rng_for(75, l), rows, cols) for l in range(batch)]
    Ws = [round_bf16(w) if dtype == "bf16" else w.astype(np.float32) for w in Ws]
    m = min(rows, cols)
    y0s = [rng_for(76, l).standard_normal(m).astype(np.float32) for l in range(batch)]
    smax = [np.linalg.svd(w.astype(np.float64), compute_uv=False)[0] for w in Ws]
    smax = [float(np.float32(s)) for s in smax]  # the fp32 value the kernel receives
    with Muon() as muon:
        y, smin = _min_singular(muon, Ws, y0s, smax, iters, dtype)
    for l in range(batch):
        ry, rs = oracle.min_singular_shifted(Ws[l].astype(np.float64), y0s[l].astype(np.float64), smax[l], iters)
        # fp32 products against fp64: a float32 replay of the same iteration stays within 1e-6
        assert abs(smin[l] - rs) <= 1e-4 * rs
        assert rel_f(y[l], ry) <= 1e-4
        assert smin[l] >= np.linalg.svd(Ws[l].astype(np.float64), compute_uv=False)[-1] * (1 - 1e-4)


def test_min_singular_full_size_in_proj_streams_in_one_launch():
    """The in_proj group of the 130M model (24 tall 3352 x 768 bf16 matrices, the one-pass
    streaming path: X X^T y = W^T W y) against the oracle's shifted iteration."""
    from spectral_optimizer_state_b200 import Muon
    rows, cols = MAMBA2_130M_IN_PROJ
    Ws = [round_bf16(weights(rng_for(78, l), rows, cols)) for l in range(24)]
    y0s = [rng_for(79, l).standard_normal(cols).astype(np.float32) for l in range(24)]
    smax = [float(np.float32(np.linalg.svd(Ws[l].astype(np.float64), compute_uv=False)[0])) if l in (0, 23)
            else 1.0 for l in range(24)]
    with Muon() as muon:
        y, smin = _min_singular(muon, Ws, y0s, smax, 16, "bf16")
    for l in (0, 23):
        ry, rs = oracle.min_singular_shifted(Ws[l].astype(np.float64), y0s[l].astype(np.float64), smax[l], 16)
        assert abs(smin[l] - rs) <= 1e-4 * rs
        assert rel_f(y[l], ry) <= 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_min_singular_full_size_out_proj_column_slabs(dtype):
    """The out_proj group of the 130M model (24 wide 768 x 1536 matrices: X = W, the one-pass
    column-slab path) against the oracle's shifted iteration, 16 steps."""
    from spectral_optimizer_state_b200 import Muon
    rows, cols = 768, 1536
    Ws = [weights(rng_for(80, l), rows, cols) for l in range(24)]
    Ws = [round_bf16(w) if dtype == "bf16" else w.astype(np.float32) for w in Ws]
    y0s = [rng_for(81, l).standard_normal(rows).astype(np.float32) for l in range(24)]
    smax = [float(np.float32(np.linalg.svd(Ws[l].astype(np.float64), compute_uv=False)[0])) if l in (0, 23)
            else 1.0 for l in range(24)]
    with Muon() as muon:
        y, smin = _min_singular(muon, Ws, y0s, smax, 16, dtype)
    for l in (0, 23):
        ry, rs = oracle.min_singular_shifted(Ws[l].astype(np.float64), y0s[l].astype(np.float64), smax[l], 16)
        assert abs(smin[l] - rs) <= 1e-4 * rs
        assert rel_f(y[l], ry) <= 1e-4


@pytest.mark.parametrize("rows,cols,batch", [(64, 64, 3), (96, 256, 2), (130, 384, 5), (1000, 4096, 1),
                                             (256, 2048, 24), (1, 64, 2), (3, 192, 2)])
def test_min_singular_column_slab_shapes(rows, cols, batch):
    """Slab widths 64 (the first four shapes; a square W is not transposed) and 256 (24 x 2048
    columns: narrower slabs would not all fit on the GPU at once; 128 is the out_proj case), rows
    not a multiple of the warps' row stride, against the oracle."""
    from spectral_optimizer_state_b200 import Muon
    Ws = [weights(rng_for(82, l), rows, cols).astype(np.float32) for l in range(batch)]
    y0s = [rng_for(83, l).standard_normal(rows).astype(np.float32) for l in range(batch)]
    smax = [float(np.float32(np.linalg.svd(w.astype(np.float64), compute_uv=False)[0])) for w in Ws]
    with Muon() as muon:
        y, smin = _min_singular(muon, Ws, y0s, smax, 12, "f32")
    for l in sorted({0, min(1, batch - 1), batch - 1}):
        ry, rs = oracle.min_singular_shifted(Ws[l].astype(np.float64), y0s[l].astype(np.float64), smax[l], 12)
        assert abs(smin[l] - rs) <= 1e-4 * rs
        assert rel_f(y[l], ry) <= 1e-4


@pytest.mark.parametrize("rows,cols", [(9, 8), (17, 16), (40, 8)])
def test_min_singular_small_tall_streaming(rows, cols):
    """Tall W with few columns on the streaming shifted path: a stage of fewer than eight rows,
    one block per matrix."""
    from spectral_optimizer_state_b200 import Muon
    batch = 3
    Ws = [weights(rng_for(84, l), rows, cols).astype(np.float32) for l in range(batch)]
    y0s = [rng_for(85, l).standard_normal(cols).astype(np.float32) for l in range(batch)]
    smax = [float(np.float32(np.linalg.svd(w.astype(np.float64), compute_uv=False)[0])) for w in Ws]
    with Muon() as muon:
        y, smin = _min_singular(muon, Ws, y0s, smax, 10, "f32")
    for l in range(batch):
        ry, rs = oracle.min_singular_shifted(Ws[l].astype(np.float64), y0s[l].astype(np.float64), smax[l], 10)
        assert abs(smin[l] - rs) <= 1e-4 * rs
        assert rel_f(y[l], ry) <= 1e-4


def test_min_singular_of_semi_orthogonal_is_one():
    from spectral_optimizer_state_b200 import Muon
    Q, _ = np.linalg.qr(rng_for(77, 0).standard_normal((300, 128)))
    Ws = [Q.astype(np.float32), np.ascontiguousarray(Q.T).astype(np.float32)]
    with Muon() as muon:
        _, smin_tall = _min_singular(muon, Ws[:1], [np.ones(128, np.float32)], [1.0], 5, "f32")
        _, smin_wide = _min_singular(muon, Ws[1:], [np.ones(128, np.float32)], [1.0], 5, "f32")
    assert abs(smin_tall[0] - 1.0) <= 1e-5 and abs(smin_wide[0] - 1.0) <= 1e-5


def test_spectral_plan_equals_the_methods():
    """SpectralPlan (tensors checked and marshalled once) gives what power_iteration and
    min_singular give."""
    import torch
    from spectral_optimizer_state_b200 import Muon
    Ws = [to_device(w, "bf16") for w in _spiked(160, 96, 3, 91, "bf16")]
    out = []
    with Muon() as muon:
        for use_plan in (False, True):
            u = [torch.zeros(160, device="cuda") for _ in Ws]
            v = [torch.ones(96, device="cuda") for _ in Ws]
            y = [torch.ones(96, device="cuda") for _ in Ws]
            smax = torch.zeros(3, device="cuda")
            smin = torch.zeros(3, device="cuda")
            if use_plan:
                plan = muon.spectral_plan(Ws, u, v, smax, y, smin)
                plan.power_iteration(iters=5)
                plan.min_singular(iters=7)
            else:
                muon.power_iteration(Ws, u, v, smax, iters=5)
                muon.min_singular(Ws, y, smax, smin, iters=7)
            torch.cuda.synchronize()
            out.append([t.clone() for t in u + v + y] + [smax.clone(), smin.clone()])
    for a, b in zip(*out):
        assert torch.equal(a, b)
