"""Muon for the selected projection weights, AdamW for everything else.

The protocol of "Muon Meets Mamba: Spectral Optimization for State Space
Models" (abstract) trains Mamba-2 130M with Muon on the output projections
only, the input projections only, or both, and AdamW for the rest; the
practitioner notes on the same paper (section 3.3) split the parameters by
name.  This class is the host-side bookkeeping of that split: parameters are
grouped by shape and dtype and handed to libmuon's muon_step_groups (Muon)
and muon_adamw_step (AdamW); every update runs in the library's kernels.
"""
from __future__ import annotations

from collections import OrderedDict

from .binding import MAX_BATCH, MAX_GROUPS, Muon, adamw_step


def takes_muon(name: str, shape, mode: str = "both") -> bool:
    """2-D weights whose name marks them as the selected projection group(s)."""
    if len(shape) != 2:
        return False
    if mode == "both":
        return "in_proj" in name or "out_proj" in name
    if mode in ("in_proj", "out_proj"):
        return mode in name
    if mode == "none":
        return False
    raise ValueError(f"unknown Muon selection {mode!r}")


class MuonAdamW:
    """named_params: iterable of (name, tensor) on one CUDA device."""

    def __init__(self, named_params, mode="both", device=0, coeffs=None,
                 muon_hp=None, adamw_hp=None):
        import torch
        self.mode = mode
        self.muon_hp = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True)
        self.muon_hp.update(muon_hp or {})
        self.adamw_hp = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
        self.adamw_hp.update(adamw_hp or {})
        self.ctx = Muon(device, coeffs)
        self.muon = OrderedDict()   # (shape, dtype) -> [(name, W, M)]
        self.adam = OrderedDict()   # dtype -> [(name, W, m, v)]
        for name, p in named_params:
            if takes_muon(name, tuple(p.shape), mode):
                key = (tuple(p.shape), p.dtype)
                self.muon.setdefault(key, []).append((name, p, torch.zeros(p.shape, dtype=torch.float32, device=p.device)))
            else:
                z = lambda: torch.zeros(p.numel(), dtype=torch.float32, device=p.device)  # noqa: E731
                self.adam.setdefault(p.dtype, []).append((name, p, z(), z()))
        self.t = 0
        # AdamW bias correction counts the steps each parameter actually took (a parameter
        # without a gradient in some step keeps its count, as in torch.optim.AdamW)
        self.adam_t = {n: 0 for entries in self.adam.values() for (n, _, _, _) in entries}

    def muon_names(self):
        return [n for entries in self.muon.values() for (n, _, _) in entries]

    def adamw_names(self):
        return [n for entries in self.adam.values() for (n, _, _, _) in entries]

    def step(self, grads, stream=None):
        """grads: mapping name -> gradient tensor (same shape and dtype as the parameter).

        A parameter whose name is missing from ``grads`` or maps to None (frozen, or unused
        in this backward pass) is left untouched: its weights get no decay, its Muon momentum
        no step and its AdamW moments and step count stay as they are.
        """
        self.t += 1
        groups = []
        for entries in self.muon.values():
            live = [e for e in entries if grads.get(e[0]) is not None]
            for c0 in range(0, len(live), MAX_BATCH):
                chunk = live[c0:c0 + MAX_BATCH]
                groups.append(([w for _, w, _ in chunk], [grads[n].contiguous() for n, _, _ in chunk],
                               [mbuf for _, _, mbuf in chunk]))
        for g0 in range(0, len(groups), MAX_GROUPS):
            self.ctx.step_groups(groups[g0:g0 + MAX_GROUPS], stream=stream, **self.muon_hp)
        for entries in self.adam.values():
            by_count = OrderedDict()  # one launch per distinct step count (normally exactly one)
            for e in entries:
                if grads.get(e[0]) is None:
                    continue
                self.adam_t[e[0]] += 1
                by_count.setdefault(self.adam_t[e[0]], []).append(e)
            for t, live in by_count.items():
                W = [w.view(-1) for _, w, _, _ in live]
                G = [grads[n].contiguous().view(-1) for n, _, _, _ in live]
                adamw_step(W, G, [m for _, _, m, _ in live], [v for _, _, _, v in live], t,
                           stream=stream, **self.adamw_hp)

    def state_dict(self) -> dict:
        """Optimizer state by parameter name: Muon momentum, AdamW moments, and the step count."""
        return {"t": self.t, "adamw_t": dict(self.adam_t),
                "muon": {n: m.detach().clone() for entries in self.muon.values() for (n, _, m) in entries},
                "adamw": {n: (m.detach().clone(), v.detach().clone())
                          for entries in self.adam.values() for (n, _, m, v) in entries}}

    def load_state_dict(self, state: dict):
        """Restore the state saved by ``state_dict`` for the same parameter names and shapes."""
        muon = {n: m for entries in self.muon.values() for (n, _, m) in entries}
        adam = {n: (m, v) for entries in self.adam.values() for (n, _, m, v) in entries}
        if set(state["muon"]) != set(muon) or set(state["adamw"]) != set(adam):
            raise ValueError("checkpoint holds a different parameter split")
        for n, m in state["muon"].items():
            muon[n].copy_(m)
        for n, (m, v) in state["adamw"].items():
            adam[n][0].copy_(m)
            adam[n][1].copy_(v)
        self.t = int(state["t"])
        counts = state.get("adamw_t", {n: self.t for n in adam})
        self.adam_t = {n: int(counts[n]) for n in adam}

    def close(self):
        self.ctx.close()


def torch_optimizer(named_params, mode="both", inner=None, **kw):
    """A ``torch.optim.Optimizer`` over MuonAdamW: ``step()`` reads each parameter's ``.grad``.

    named_params: (name, parameter) pairs, e.g. ``model.named_parameters()``.  Parameters whose
    ``.grad`` is None at ``step()`` are skipped, as ``torch.optim.AdamW`` skips them: no decay,
    no momentum step, no moment update.  ``inner`` replaces the MuonAdamW instance (host-side
    tests only).
    """
    import torch

    named = [(n, p) for n, p in named_params]

    class MuonAdamWOptimizer(torch.optim.Optimizer):
        def __init__(self):
            super().__init__([p for _, p in named], defaults={})
            self.inner = inner if inner is not None else MuonAdamW(named, mode=mode, **kw)
            self.names = [n for n, _ in named]

        @torch.no_grad()
        def step(self, closure=None):
            loss = None
            if closure is not None:
                with torch.enable_grad():
                    loss = closure()
            grads = {n: p.grad for n, p in named}
            self.inner.step(grads)
            return loss

        def state_dict(self):
            return self.inner.state_dict()

        def load_state_dict(self, state):
            self.inner.load_state_dict(state)

    return MuonAdamWOptimizer()
