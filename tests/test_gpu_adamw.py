"""AdamW kernel and the Muon/AdamW parameter split vs the fp64 oracles (needs a B200)."""
import numpy as np
import pytest

import oracle
from synthetic import group_inputs, rng_for, round_bf16
from tests.gpu_common import F32_TOL, half_ulp_bf16, rel_f, to_numpy

pytestmark = pytest.mark.gpu

AHP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
SHAPES = [(50280 // 8, 768), (1536,), (1792, 1, 4), (24,), (37, 53), (4097,)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_adamw_matches_oracle_three_steps(dtype):
    import torch
    from spectral_optimizer_state_b200 import adamw_step
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    rng = rng_for(61, 0)
    W0 = [rng.standard_normal(s).astype(np.float32) * 0.02 for s in SHAPES]
    if dtype == "bf16":
        W0 = [round_bf16(w) for w in W0]
    W = [torch.from_numpy(w).to(tdt).cuda() for w in W0]
    m = [torch.zeros(w.size, dtype=torch.float32, device="cuda") for w in W0]
    v = [torch.zeros(w.size, dtype=torch.float32, device="cuda") for w in W0]
    ref = [(w.astype(np.float64), np.zeros(w.shape), np.zeros(w.shape)) for w in W0]
    for t in range(1, 4):
        G = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
        if dtype == "bf16":
            G = [round_bf16(g) for g in G]
        adamw_step([w.view(-1) for w in W], [torch.from_numpy(g).to(tdt).cuda().view(-1) for g in G], m, v, t, **AHP)
        ref = [oracle.adamw_step(r[0], g.astype(np.float64), r[1], r[2], t, **AHP) for r, g in zip(ref, G)]
    torch.cuda.synchronize()
    for w, w0, a, b, (rw, rm, rv) in zip(W, W0, m, v, ref):
        assert rel_f(to_numpy(a).reshape(rm.shape), rm) <= 1e-5
        assert rel_f(to_numpy(b).reshape(rv.shape), rv) <= 1e-5
        dW = rw - w0
        if dtype == "f32":
            assert rel_f(to_numpy(w) - w0, dW) <= F32_TOL
        else:
            bound = 2e-2 * np.linalg.norm(dW) + np.linalg.norm(half_ulp_bf16(rw))
            assert np.linalg.norm(to_numpy(w) - rw) <= bound


@pytest.mark.parametrize("mode", ["out_proj", "in_proj", "both"])
def test_muon_adamw_split_small_mamba_like(mode):
    """A 2-layer Mamba-2-like parameter set (reduced widths): each parameter is
    updated by the optimizer its name selects, matching that optimizer's oracle."""
    import torch
    from spectral_optimizer_state_b200 import MuonAdamW
    names = []
    for layer in range(2):
        pre = f"layers.{layer}.mixer."
        names += [(pre + "in_proj.weight", (424, 96)), (pre + "out_proj.weight", (96, 192)),
                  (pre + "conv1d.weight", (224, 1, 4)), (pre + "A_log", (3,)), (pre + "D", (3,)),
                  (f"layers.{layer}.norm.weight", (96,))]
    names.append(("embeddings.weight", (500, 96)))
    rng = rng_for(62, 0)
    params, W0 = [], {}
    for n, s in names:
        w = round_bf16(rng.standard_normal(s).astype(np.float32) * 0.02)
        W0[n] = w
        params.append((n, torch.from_numpy(w).to(torch.bfloat16).cuda()))
    opt = MuonAdamW(params, mode=mode, coeffs=[oracle.QUINTIC] * 5)
    assert set(opt.muon_names()) == {n for n, s in names if oracle.select_muon(n, s, mode)}
    G = {n: round_bf16(rng.standard_normal(s).astype(np.float32)) for n, s in names}
    opt.step({n: torch.from_numpy(g).to(torch.bfloat16).cuda() for n, g in G.items()})
    torch.cuda.synchronize()
    for n, w in params:
        g = G[n].astype(np.float64)
        if oracle.select_muon(n, W0[n].shape, mode):
            r = oracle.muon_step(W0[n], g, np.zeros(g.shape), [oracle.QUINTIC] * 5, **opt.muon_hp)
            ref = r["W"]
        else:
            ref, _, _ = oracle.adamw_step(W0[n], g, np.zeros(g.shape), np.zeros(g.shape), 1, **opt.adamw_hp)
        bound = 2e-2 * np.linalg.norm(ref - W0[n]) + np.linalg.norm(half_ulp_bf16(ref))
        assert np.linalg.norm(to_numpy(w) - ref) <= bound, n
    opt.close()


def test_muon_adamw_checkpoint_resume_equals_straight_run():
    """Three steps straight equal two steps, a state_dict round trip into a new optimizer, one more."""
    import io
    import torch
    from spectral_optimizer_state_b200 import MuonAdamW
    names = [("layers.0.mixer.in_proj.weight", (424, 96)), ("layers.0.mixer.out_proj.weight", (96, 192)),
             ("layers.0.mixer.A_log", (3,)), ("embeddings.weight", (500, 96))]
    rng = rng_for(63, 0)
    W0 = {n: round_bf16(rng.standard_normal(s).astype(np.float32) * 0.02) for n, s in names}
    Gs = [{n: torch.from_numpy(round_bf16(rng.standard_normal(s).astype(np.float32))).to(torch.bfloat16).cuda()
           for n, s in names} for _ in range(3)]

    def fresh():
        params = [(n, torch.from_numpy(W0[n]).to(torch.bfloat16).cuda()) for n, _ in names]
        return params, MuonAdamW(params, mode="both", coeffs=[oracle.QUINTIC] * 5)

    pa, a = fresh()
    for g in Gs:
        a.step(g)
    pb, b = fresh()
    for g in Gs[:2]:
        b.step(g)
    buf = io.BytesIO()
    torch.save({"params": {n: w.cpu() for n, w in pb}, "opt": b.state_dict()}, buf)
    b.close()
    buf.seek(0)
    ck = torch.load(buf)
    pc = [(n, ck["params"][n].cuda()) for n, _ in names]
    c = MuonAdamW(pc, mode="both", coeffs=[oracle.QUINTIC] * 5)
    c.load_state_dict(ck["opt"])
    c.step(Gs[2])
    torch.cuda.synchronize()
    for (n, wa), (_, wc) in zip(pa, pc):
        assert torch.equal(wa, wc), n
    a.close()
    c.close()
