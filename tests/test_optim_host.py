"""The torch.optim wrapper hands every parameter's gradient, by name, to the optimizer (no GPU)."""
import torch

from spectral_optimizer_state_b200 import takes_muon, torch_optimizer


class _Recorder:
    def __init__(self):
        self.calls = []
        self.state = {"t": 0}

    def step(self, grads):
        self.calls.append({n: g.clone() for n, g in grads.items()})
        self.state["t"] += 1

    def state_dict(self):
        return dict(self.state)

    def load_state_dict(self, st):
        self.state = dict(st)


def test_wrapper_passes_named_gradients_and_zero_grad_works():
    model = torch.nn.ModuleDict({"in_proj": torch.nn.Linear(8, 16, bias=False),
                                 "norm": torch.nn.LayerNorm(16)})
    rec = _Recorder()
    opt = torch_optimizer(model.named_parameters(), inner=rec)
    x = torch.randn(4, 8)
    loss = model["norm"](model["in_proj"](x)).pow(2).sum()
    loss.backward()
    got = opt.step()
    assert got is None and len(rec.calls) == 1
    call = rec.calls[0]
    assert set(call) == {n for n, _ in model.named_parameters()}
    for n, p in model.named_parameters():
        assert torch.equal(call[n], p.grad)
    opt.zero_grad()
    assert all(p.grad is None or not p.grad.any() for p in model.parameters())
    opt.step()  # missing gradients become zeros
    assert all(not g.any() for g in rec.calls[1].values())
    assert opt.state_dict() == {"t": 2}
    opt.load_state_dict({"t": 5})
    assert rec.state == {"t": 5}


def test_closure_is_evaluated_with_gradients():
    w = torch.nn.Parameter(torch.ones(3, 3))
    rec = _Recorder()
    opt = torch_optimizer([("out_proj.weight", w)], inner=rec)

    def closure():
        opt.zero_grad()
        loss = (w * 2).sum()
        loss.backward()
        return loss

    loss = opt.step(closure)
    assert float(loss.detach()) == 18.0
    assert torch.equal(rec.calls[0]["out_proj.weight"], torch.full((3, 3), 2.0))
    assert takes_muon("out_proj.weight", (3, 3))
