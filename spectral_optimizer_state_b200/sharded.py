"""Data-parallel Muon with the optimizer state sharded by matrix ownership.

Each matrix's Muon step is independent of every other matrix (Muon Meets
Mamba: Spectral Optimization for State Space Models, abstract: Muon
orthogonalises the update of each weight matrix on its own).  With N
data-parallel ranks that each hold a full gradient, one step is therefore

  1. reduce-scatter of the gradients: rank r receives the sum, over ranks, of
     the gradients of the matrices it owns (the 1/N of the average is folded
     into the momentum pass as libmuon's gradient scale, not a separate pass);
  2. the local Muon step (momentum, Newton-Schulz, apply) on the owned
     matrices only, through libmuon;
  3. all-gather of the updated weights, so every rank holds the new W.

The momentum buffers exist only on the owner, so the fp32 optimizer state per
GPU is 1/N of the model's.  Ownership balances the algorithmic Newton-Schulz
flops (3 m^2 n + m^3 per iteration on the wide m x n view) with a greedy
longest-processing-time assignment.

Weights and gradients live in two flat buffers laid out owner-major: rank r's
matrices are contiguous in segment r, and every segment is padded to the
largest one.  The caller's weight and gradient tensors are views into them,
so both collectives run in place with no packing copies:
``reduce_scatter_tensor(G[r], G)`` and ``all_gather_into_tensor(W, W[r])``.
Every matrix starts on a 256-byte boundary, which keeps libmuon's vector
paths and TMA descriptors valid for the views.
"""
from __future__ import annotations

from typing import Callable, Sequence

ALIGN_ELEMS = 128  # 256 bytes of bf16, 512 of fp32


def ns_cost(rows: int, cols: int) -> int:
    """Algorithmic Newton-Schulz flops of one iteration on the wide view (m = min, n = max)."""
    m, n = min(rows, cols), max(rows, cols)
    return 3 * m * m * n + m ** 3


def partition(shapes: Sequence[tuple], world: int) -> list[int]:
    """Owner rank of each matrix: largest cost first, to the least-loaded rank (ties: lower index, lower rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda i: (-ns_cost(*shapes[i]), i))
    load = [0] * world
    owner = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += ns_cost(*shapes[i])
    return owner


def _round_up(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def layout(shapes: Sequence[tuple], owner: Sequence[int], world: int):
    """(offset of each matrix in the flat buffer, padded segment length S); segment r is [r*S, (r+1)*S)."""
    used = [0] * world
    local = [0] * len(shapes)
    for i, (r, c) in enumerate(shapes):
        o = owner[i]
        local[i] = used[o]
        used[o] += _round_up(r * c, ALIGN_ELEMS)
    seg = max(max(used), ALIGN_ELEMS)
    return [owner[i] * seg + local[i] for i in range(len(shapes))], seg


def _libmuon_step(device):
    from .binding import Muon
    mu = Muon(device)

    def step(groups, hp, stream=None):
        mu.step_groups(groups, stream=stream, **hp)

    step.muon = mu
    return step


class ShardedMuon:
    """Muon over N data-parallel ranks with matrix-owner sharding of the momentum state.

    shapes: (rows, cols) of every 2-D weight, the same list on every rank.
    weights / grads: views (one per shape) into the flat weight / gradient
    buffers; write each step's local gradient into ``grads[i]`` and read the
    model's weights from ``weights[i]``.  ``local_step(groups, hp)`` performs
    Muon steps on [(W list, G list, M list), ...] same-shape groups, reading each
    G as ``hp["grad_scale"] * G``; it defaults to libmuon on this rank's GPU and is
    replaceable only for host-side tests.
    """

    def __init__(self, shapes: Sequence[tuple], dtype=None, device=None, process_group=None,
                 coeffs: Sequence | None = None, local_step: Callable | None = None, state_dtype=None, **hp):
        import torch
        import torch.distributed as dist
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        if any(len(s) != 2 for s in self.shapes):
            raise ValueError("ShardedMuon takes 2-D weights only")
        self.group = process_group
        self.world = dist.get_world_size(process_group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(process_group) if dist.is_initialized() else 0
        self.dtype = dtype if dtype is not None else torch.bfloat16
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.hp = dict(hp)
        self.owner = partition(self.shapes, self.world)
        self.offsets, self.seg = layout(self.shapes, self.owner, self.world)
        n = self.world * self.seg
        self.flat_w = torch.zeros(n, dtype=self.dtype, device=self.device)
        self.flat_g = torch.zeros(n, dtype=self.dtype, device=self.device)
        self.weights = [self._view(self.flat_w, i) for i in range(len(self.shapes))]
        self.grads = [self._view(self.flat_g, i) for i in range(len(self.shapes))]
        self.owned = [i for i in range(len(self.shapes)) if self.owner[i] == self.rank]
        sdt = state_dtype if state_dtype is not None else torch.float32  # libmuon keeps M in fp32
        self.momenta = {i: torch.zeros(self.shapes[i], dtype=sdt, device=self.device) for i in self.owned}
        if local_step is None:
            local_step = _libmuon_step(self.device.index or 0)
            if coeffs is not None:
                local_step.muon.set_coeffs(coeffs)
        self.local_step = local_step
        # owned matrices grouped by shape, index order inside a group
        by_shape: dict[tuple, list[int]] = {}
        for i in self.owned:
            by_shape.setdefault(self.shapes[i], []).append(i)
        self._groups = list(by_shape.values())

    def _view(self, flat, i):
        r, c = self.shapes[i]
        o = self.offsets[i]
        return flat[o:o + r * c].view(r, c)

    def segment(self, flat, rank=None):
        r = self.rank if rank is None else rank
        return flat[r * self.seg:(r + 1) * self.seg]

    def load_weights(self, tensors: Sequence):
        """Copy initial weights (identical on every rank) into the flat buffer."""
        for dst, src in zip(self.weights, tensors):
            dst.copy_(src)

    def owned_bytes(self) -> dict:
        """Optimizer-state and exchange bytes of this rank (for reports)."""
        e = self.flat_w.element_size()
        return {"momentum_bytes": 4 * sum(self.shapes[i][0] * self.shapes[i][1] for i in self.owned),
                "reduce_scatter_bytes": self.world * self.seg * e,
                "all_gather_bytes": self.world * self.seg * e}

    def state_dict(self) -> dict:
        """This rank's optimizer state: its momentum buffers by matrix index, and the ownership they follow.

        Save one per rank (e.g. ``torch.save(opt.state_dict(), f"muon_rank{rank}.pt")``); the
        weights are the model's and are saved with it.
        """
        return {"shapes": list(self.shapes), "world": self.world, "owner": list(self.owner),
                "momenta": {i: m.detach().clone() for i, m in self.momenta.items()}}

    def load_state_dict(self, state: dict):
        """Restore the momentum buffers saved by ``state_dict`` on the same rank of a job with the
        same shapes and world size (ownership is a pure function of both, so it matches)."""
        if [tuple(x) for x in state["shapes"]] != self.shapes or state["world"] != self.world:
            raise ValueError("checkpoint was written for different shapes or a different world size")
        if list(state["owner"]) != self.owner:
            raise ValueError("checkpoint ownership differs from this job's")
        if sorted(state["momenta"]) != sorted(self.momenta):
            raise ValueError("checkpoint holds another rank's matrices")
        for i, m in state["momenta"].items():
            self.momenta[i].copy_(m)

    def step(self, stream=None, mark=None):
        """One data-parallel Muon step: reduce-scatter G, local step on owned matrices, all-gather W.

        ``mark(phase)``, if given, is called before each part ("reduce_scatter", "local_step",
        "all_gather") and at the end ("end"), e.g. to record CUDA events for a per-part timing.
        """
        import torch.distributed as dist
        mark = mark or (lambda phase: None)
        mine_g = self.segment(self.flat_g)
        mark("reduce_scatter")
        if self.world > 1:
            dist.reduce_scatter_tensor(mine_g, self.flat_g, op=dist.ReduceOp.SUM, group=self.group)
        groups = [([self.weights[i] for i in idx], [self.grads[i] for i in idx], [self.momenta[i] for i in idx])
                  for idx in self._groups]
        mark("local_step")
        if groups:
            # the owned gradients hold the SUM over ranks; the step reads grad_scale * G
            self.local_step(groups, dict(self.hp, grad_scale=1.0 / self.world), stream)
        mark("all_gather")
        if self.world > 1:
            dist.all_gather_into_tensor(self.flat_w, self.segment(self.flat_w), group=self.group)
        mark("end")
