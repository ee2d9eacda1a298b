"""ShardedMuon on one GPU (no collectives) runs the same kernels as a plain grouped step (needs a B200)."""
import numpy as np
import pytest

from synthetic import gaussian_spike, rng_for, round_bf16, weights

pytestmark = pytest.mark.gpu

SHAPES = [(192, 320), (320, 192), (192, 320), (77, 45), (320, 192)]


def test_sharded_world_one_equals_plain_grouped_step_bitwise():
    import torch
    from spectral_optimizer_state_b200 import Muon
    from spectral_optimizer_state_b200.sharded import ShardedMuon
    hp = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True, scale_mode=0)
    W0 = [torch.from_numpy(round_bf16(weights(rng_for(600, i), r, c))).to(torch.bfloat16).cuda()
          for i, (r, c) in enumerate(SHAPES)]
    opt = ShardedMuon(SHAPES, dtype=torch.bfloat16, device="cuda", **hp)
    opt.load_weights(W0)
    Wp = [w.clone() for w in W0]
    Mp = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in SHAPES]
    by_shape = {}
    for i, s in enumerate(SHAPES):
        by_shape.setdefault(s, []).append(i)
    with Muon() as mu:
        for step in range(3):
            G = [torch.from_numpy(round_bf16(gaussian_spike(rng_for(601 + step, i), r, c))).to(torch.bfloat16).cuda()
                 for i, (r, c) in enumerate(SHAPES)]
            for g, src in zip(opt.grads, G):
                g.copy_(src)
            opt.step()
            mu.step_groups([([Wp[i] for i in idx], [G[i] for i in idx], [Mp[i] for i in idx])
                            for idx in by_shape.values()], **hp)
    torch.cuda.synchronize()
    for i in range(len(SHAPES)):
        assert torch.equal(opt.weights[i], Wp[i])
        assert torch.equal(opt.momenta[i], Mp[i])
    assert opt.local_step.muon.status()[0] == 0


def test_gradient_scale_equals_prescaled_gradients_bitwise():
    """grad_scale = 1/2 on G gives exactly what grad_scale = 1 gives on G/2 (halving is exact in
    bf16 and fp32), so the data-parallel 1/N average folded into the momentum pass changes nothing
    but the extra pass; a zero scale (an uninitialised field) is rejected."""
    import torch
    from spectral_optimizer_state_b200 import Muon, MuonError
    shape = (320, 192)
    G = [torch.from_numpy(round_bf16(gaussian_spike(rng_for(650, i), *shape))).to(torch.bfloat16).cuda()
         for i in range(3)]
    W0 = [torch.from_numpy(round_bf16(weights(rng_for(651, i), *shape))).to(torch.bfloat16).cuda() for i in range(3)]
    out = []
    with Muon() as mu:
        for gs, Gs in ((0.5, G), (1.0, [g / 2 for g in G])):
            W = [w.clone() for w in W0]
            M = [torch.zeros(shape, device="cuda") for _ in range(3)]
            for _ in range(2):
                mu.step(W, Gs, M, grad_scale=gs)
            assert mu.status()[0] == 0
            out.append((W, M))
        with pytest.raises(MuonError):
            mu.step([w.clone() for w in W0], G, [torch.zeros(shape, device="cuda") for _ in range(3)], grad_scale=0.0)
    for a, b in zip(out[0][0] + out[0][1], out[1][0] + out[1][1]):
        assert torch.equal(a, b)
