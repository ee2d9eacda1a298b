"""CUDA-graph capture of the library's stream-ordered calls (needs a B200).

A training loop may capture its optimizer step into a CUDA graph and replay it.  Once the
context's buffers are sized (one call of the same shapes before capture), a step plan and a
spectral plan queue only memsets and kernel launches, so the captured graph replays the same
work: the tensors stepped by replays must equal, bit for bit, a twin set stepped by eager calls
on the same inputs.  A call that would have to grow the context while its stream is capturing is
refused with MUON_ERR_ALLOC before anything is queued, and the capture stays usable.
"""
import pytest

import oracle
from synthetic import (MAMBA2_130M_IN_PROJ, MAMBA2_130M_OUT_PROJ, gaussian_spike, group_inputs, group_weights,
                       rng_for, round_bf16)
from tests.gpu_common import to_device

pytestmark = pytest.mark.gpu

HP = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7)
MUON_ERR_ALLOC = 8


def _twin_groups(shapes, batch, config):
    """Two identical sets of (W, M) per group and one set of gradient buffers both read."""
    import torch
    W0 = [[to_device(w, "bf16") for w in group_weights(config, i, batch, *sh)] for i, sh in enumerate(shapes)]
    Wa = [[w.clone() for w in ws] for ws in W0]
    Wb = [[w.clone() for w in ws] for ws in W0]
    Ma = [[torch.zeros(sh, device="cuda") for _ in range(batch)] for sh in shapes]
    Mb = [[torch.zeros(sh, device="cuda") for _ in range(batch)] for sh in shapes]
    G = [[torch.empty(sh, dtype=torch.bfloat16, device="cuda") for _ in range(batch)] for sh in shapes]
    return Wa, Ma, Wb, Mb, G


def _load_grads(G, shapes, batch, config, step):
    """Copy this step's seeded gradients into the fixed gradient buffers (the graph reads them)."""
    import torch
    for i, sh in enumerate(shapes):
        for l, g in enumerate(group_inputs(config, step, i, batch, *sh)):
            G[i][l].copy_(torch.from_numpy(round_bf16(g)).to(torch.bfloat16))


@pytest.mark.parametrize("case", ["small", "mamba2_130m"])
def test_step_plan_replays_in_cuda_graph(case):
    """Replays of a captured step plan, each on fresh gradients, equal eager steps bitwise."""
    import torch
    from spectral_optimizer_state_b200 import Muon
    if case == "small":
        shapes, batch, config, steps = [(200, 328), (328, 200)], 2, 8, 4
    else:
        shapes, batch, config, steps = [MAMBA2_130M_IN_PROJ, MAMBA2_130M_OUT_PROJ], 24, 1, 3
    Wa, Ma, Wb, Mb, G = _twin_groups(shapes, batch, config)
    w_start = Wb[0][0].clone()
    with Muon(0) as muon:
        muon.set_coeffs([oracle.QUINTIC] * 5)
        plan = muon.step_plan([(Wb[i], G[i], Mb[i]) for i in range(len(shapes))], **HP)
        _load_grads(G, shapes, batch, config, 0)
        muon.step_groups([(Wa[i], G[i], Ma[i]) for i in range(len(shapes))], **HP)
        plan()  # sizes the context's buffers before capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            plan()
        for step in range(1, steps + 1):
            _load_grads(G, shapes, batch, config, step)
            muon.step_groups([(Wa[i], G[i], Ma[i]) for i in range(len(shapes))], **HP)
            graph.replay()
        torch.cuda.synchronize()
        assert muon.status()[0] == 0
        del graph
    for xa, xb in zip([w for ws in Wa + Ma for w in ws], [w for ws in Wb + Mb for w in ws]):
        assert torch.equal(xa, xb)
    assert not torch.equal(Wb[0][0], w_start)  # the replays really stepped


def test_capture_refuses_growth_and_keeps_the_capture():
    """On a fresh context the first step must grow the workspace: made while the stream captures,
    it is refused (MUON_ERR_ALLOC) with nothing queued, and the rest of the capture replays."""
    import torch
    from spectral_optimizer_state_b200 import Muon, MuonError
    shapes, batch, config = [(200, 328)], 2, 9
    Wa, Ma, Wb, Mb, G = _twin_groups(shapes, batch, config)
    _load_grads(G, shapes, batch, config, 0)
    x = torch.zeros(1024, device="cuda")
    with Muon(0) as muon:
        plan = muon.step_plan([(Wb[0], G[0], Mb[0])], **HP)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        refused = None
        with torch.cuda.graph(graph):
            try:
                plan()
            except MuonError as e:
                refused = e
            x.add_(1.0)
        assert refused is not None and refused.status == MUON_ERR_ALLOC
        assert "capturing" in str(refused)
        graph.replay()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(x, torch.full_like(x, 2.0))
        del graph
        # the refused call changed nothing; made outside capture it steps as usual
        assert torch.equal(Wa[0][0], Wb[0][0]) and torch.equal(Mb[0][0], Ma[0][0])
        plan()
        muon.step_groups([(Wa[0], G[0], Ma[0])], **HP)
        torch.cuda.synchronize()
        assert muon.status()[0] == 0
    for xa, xb in zip(Wa[0] + Ma[0], Wb[0] + Mb[0]):
        assert torch.equal(xa, xb)


@pytest.mark.parametrize("rows,cols,batch", [(160, 96, 3), (96, 256, 2), MAMBA2_130M_IN_PROJ + (24,),
                                             MAMBA2_130M_OUT_PROJ + (24,)])
def test_spectral_plan_replays_in_cuda_graph(rows, cols, batch):
    """Power iteration and the smallest-singular-value iteration (cooperative launches) captured
    once and replayed continue exactly as eager calls do."""
    import torch
    from spectral_optimizer_state_b200 import Muon
    W = [to_device(round_bf16(gaussian_spike(rng_for(93, l), rows, cols, rank=1)), "bf16") for l in range(batch)]
    m = min(rows, cols)

    def vectors():
        return ([torch.zeros(rows, device="cuda") for _ in W], [torch.ones(cols, device="cuda") for _ in W],
                [torch.ones(m, device="cuda") for _ in W], torch.zeros(batch, device="cuda"),
                torch.zeros(batch, device="cuda"))

    a, b = vectors(), vectors()
    with Muon(0) as muon:
        # spectral_plan(W, u, v, sigma, y, sigma_min); vectors() is (u, v, y, sigma, sigma_min)
        pa = muon.spectral_plan(W, a[0], a[1], a[3], a[2], a[4])
        pb = muon.spectral_plan(W, b[0], b[1], b[3], b[2], b[4])
        for p in (pa, pb):  # sizes the scratch before capture
            p.power_iteration(iters=4)
            p.min_singular(iters=6)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            pb.power_iteration(iters=4)
            pb.min_singular(iters=6)
        for _ in range(2):
            pa.power_iteration(iters=4)
            pa.min_singular(iters=6)
            graph.replay()
        torch.cuda.synchronize()
        assert muon.status()[0] == 0
        del graph
    for xa, xb in zip(a[0] + a[1] + a[2] + [a[3], a[4]], b[0] + b[1] + b[2] + [b[3], b[4]]):
        assert torch.equal(xa, xb)
    assert float(b[3][0]) > 0.0 and float(b[4][0]) > 0.0


def test_captured_context_never_regrows():
    """After a capture the graph holds the context's buffers: a later eager call that would need
    larger ones is refused (MUON_ERR_ALLOC) and the graph keeps replaying correctly."""
    import torch
    from spectral_optimizer_state_b200 import Muon, MuonError
    shapes, batch, config = [(200, 328)], 2, 10
    Wa, Ma, Wb, Mb, G = _twin_groups(shapes, batch, config)
    _load_grads(G, shapes, batch, config, 0)
    big = _twin_groups([(512, 700)], 2, config)
    with Muon(0) as muon:
        plan = muon.step_plan([(Wb[0], G[0], Mb[0])], **HP)
        plan()
        muon.step_groups([(Wa[0], G[0], Ma[0])], **HP)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            plan()
        with pytest.raises(MuonError) as info:
            muon.step_groups([(big[0][0], big[4][0], big[1][0])], **HP)
        assert info.value.status == MUON_ERR_ALLOC and "graph" in str(info.value)
        for step in (1, 2):
            _load_grads(G, shapes, batch, config, step)
            muon.step_groups([(Wa[0], G[0], Ma[0])], **HP)
            graph.replay()
        torch.cuda.synchronize()
        assert muon.status()[0] == 0
        del graph
    for xa, xb in zip(Wa[0] + Ma[0], Wb[0] + Mb[0]):
        assert torch.equal(xa, xb)
