"""The torch.optim wrapper hands every parameter's gradient, by name, to the optimizer (no GPU)."""
import torch

from spectral_optimizer_state_b200 import takes_muon, torch_optimizer


class _Recorder:
    def __init__(self):
        self.calls = []
        self.state = {"t": 0}

    def step(self, grads):
        self.calls.append({n: (None if g is None else g.clone()) for n, g in grads.items()})
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
    assert all(p.grad is None for p in model.parameters())
    opt.step()  # no gradient: passed on as None, so the optimizer skips the parameter
    assert all(g is None for g in rec.calls[1].values())
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


class _FakeCtx:
    """Stands in for the libmuon context: records which weights each Muon call would update."""

    def __init__(self, *a, **k):
        self.calls = []

    def step_groups(self, groups, stream=None, **hp):
        self.calls.append([[w.data_ptr() for w in W] for (W, G, M) in groups])

    def close(self):
        pass


def test_parameters_without_gradients_are_left_untouched(monkeypatch):
    """A frozen parameter (or one unused in this backward) gets no decay, no momentum step and no
    AdamW moment update; AdamW's bias correction counts only the steps a parameter took."""
    from spectral_optimizer_state_b200 import optim
    adam_calls = []

    def fake_adamw(W, G, m, v, step, stream=None, **hp):
        adam_calls.append(([w.data_ptr() for w in W], step))

    monkeypatch.setattr(optim, "Muon", _FakeCtx)
    monkeypatch.setattr(optim, "adamw_step", fake_adamw)
    params = {"l0.in_proj.weight": torch.zeros(6, 4), "l1.in_proj.weight": torch.zeros(6, 4),
              "l0.norm.weight": torch.zeros(4), "l1.norm.weight": torch.zeros(4)}
    opt = optim.MuonAdamW(list(params.items()))
    grads = {n: torch.ones_like(p) for n, p in params.items()}
    frozen = {"l1.in_proj.weight", "l1.norm.weight"}
    opt.step({n: (None if n in frozen else g) for n, g in grads.items()})
    muon_ptrs = [ptr for call in opt.ctx.calls for grp in call for ptr in grp]
    assert muon_ptrs == [params["l0.in_proj.weight"].data_ptr()]
    assert adam_calls == [([params["l0.norm.weight"].data_ptr()], 1)]
    # every parameter steps next: the frozen AdamW parameter takes its first step (count 1),
    # the other its second, in separate launches
    adam_calls.clear()
    opt.step(grads)
    assert sorted(adam_calls, key=lambda c: c[1]) == [([params["l1.norm.weight"].data_ptr()], 1),
                                                      ([params["l0.norm.weight"].data_ptr()], 2)]
    assert len(opt.ctx.calls[-1][0]) == 2  # both in_proj matrices in one Muon group
    st = opt.state_dict()
    assert st["t"] == 2 and st["adamw_t"] == {"l0.norm.weight": 2, "l1.norm.weight": 1}
