"""Matrix-owner sharding of the Muon step: partition, layout and the gloo (CPU) data-parallel path."""
import os
import socket

import numpy as np
import pytest

import oracle
from spectral_optimizer_state_b200.sharded import ALIGN_ELEMS, layout, ns_cost, partition
from synthetic import MAMBA2_130M_IN_PROJ, MAMBA2_130M_OUT_PROJ, gaussian_spike, rng_for, weights

HP = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True, scale_mode=0)
COEFFS = [oracle.QUINTIC] * 5
SHAPES = [(48, 80), (80, 48), (48, 80), (33, 20), (64, 64), (80, 48), (20, 33)]


def test_partition_balances_the_130m_model_on_eight_ranks():
    shapes = [MAMBA2_130M_IN_PROJ] * 24 + [MAMBA2_130M_OUT_PROJ] * 24
    owner = partition(shapes, 8)
    for r in range(8):
        mine = [shapes[i] for i in range(48) if owner[i] == r]
        assert mine.count(MAMBA2_130M_IN_PROJ) == 3 and mine.count(MAMBA2_130M_OUT_PROJ) == 3
    assert partition(shapes, 8) == owner  # deterministic
    assert partition(shapes, 1) == [0] * 48


def test_partition_is_lpt_within_its_bound():
    rng = rng_for(5, 0)
    shapes = [tuple(int(x) for x in rng.integers(16, 600, 2)) for _ in range(37)]
    for world in (2, 3, 5):
        owner = partition(shapes, world)
        load = [sum(ns_cost(*shapes[i]) for i in range(37) if owner[i] == r) for r in range(world)]
        # Graham's bound for LPT: makespan <= (4/3 - 1/(3 world)) * optimum, optimum >= max(mean, largest)
        lower = max(sum(load) / world, max(ns_cost(*s) for s in shapes))
        assert max(load) <= (4 / 3 - 1 / (3 * world)) * lower + 1e-9


def test_layout_is_owner_major_aligned_and_disjoint():
    owner = partition(SHAPES, 3)
    off, seg = layout(SHAPES, owner, 3)
    spans = sorted((o, o + r * c, owner[i]) for i, ((r, c), o) in enumerate(zip(SHAPES, off)))
    for (a0, a1, ra), (b0, b1, rb) in zip(spans, spans[1:]):
        assert a1 <= b0
    for i, (r, c) in enumerate(SHAPES):
        assert off[i] % ALIGN_ELEMS == 0
        assert owner[i] * seg <= off[i] and off[i] + r * c <= (owner[i] + 1) * seg
    assert seg % ALIGN_ELEMS == 0


def _oracle_step(groups, hp, stream=None):
    """Stand-in for libmuon's step on CPU: reads G as grad_scale * G, as the library does."""
    import torch
    hp = dict(hp)
    gs = hp.pop("grad_scale", 1.0)
    for Ws, Gs, Ms in groups:
        for W, G, M in zip(Ws, Gs, Ms):
            r = oracle.muon_step(W.numpy(), gs * G.numpy(), M.numpy(), COEFFS, **hp)
            W.copy_(torch.from_numpy(r["W"]))
            M.copy_(torch.from_numpy(r["M"]))


def _grads(rank, step):
    return [gaussian_spike(rng_for(900 + 10 * step + rank, i), r, c, rank=2) for i, (r, c) in enumerate(SHAPES)]


def _worker(rank, world, port, steps, q):
    import torch
    import torch.distributed as dist
    from spectral_optimizer_state_b200.sharded import ShardedMuon
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = ShardedMuon(SHAPES, dtype=torch.float64, device="cpu", local_step=_oracle_step,
                          state_dtype=torch.float64, **HP)
        opt.load_weights([torch.from_numpy(weights(rng_for(800, i), r, c)) for i, (r, c) in enumerate(SHAPES)])
        for s in range(steps):
            for g, G in zip(opt.grads, _grads(rank, s)):
                g.copy_(torch.from_numpy(G))
            opt.step()
        q.put((rank, [w.numpy().copy() for w in opt.weights], sorted(opt.momenta), opt.owner))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2])
def test_sharded_step_matches_single_process_oracle_on_averaged_gradients(world):
    import torch.multiprocessing as mp
    steps = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, steps, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort(key=lambda t: t[0])
    # reference: one process, gradients averaged over the ranks
    W = [weights(rng_for(800, i), r, c) for i, (r, c) in enumerate(SHAPES)]
    M = [np.zeros(s) for s in SHAPES]
    for s in range(steps):
        per_rank = [_grads(r, s) for r in range(world)]
        for i in range(len(SHAPES)):
            G = sum(per_rank[r][i] for r in range(world)) / world
            res = oracle.muon_step(W[i], G, M[i], COEFFS, **HP)
            W[i], M[i] = res["W"], res["M"]
    owner = out[0][3]
    for rank, Ws, owned, own in out:
        assert own == owner
        assert owned == [i for i in range(len(SHAPES)) if owner[i] == rank]  # momentum only on the owner
        for i in range(len(SHAPES)):
            # the sum of two fp64 gradients then * 1/2 vs (a + b) / 2: equal up to one rounding
            assert np.allclose(Ws[i], W[i], rtol=0, atol=1e-12)
    if world == 2:
        assert set(owner) == {0, 1}


def _resume_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from spectral_optimizer_state_b200.sharded import ShardedMuon
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def make():
            return ShardedMuon(SHAPES, dtype=torch.float64, device="cpu", local_step=_oracle_step,
                               state_dtype=torch.float64, **HP)

        W0 = [torch.from_numpy(weights(rng_for(800, i), r, c)) for i, (r, c) in enumerate(SHAPES)]

        def run(opt, first, last):
            for s in range(first, last):
                for g, G in zip(opt.grads, _grads(rank, s)):
                    g.copy_(torch.from_numpy(G))
                opt.step()

        straight = make()
        straight.load_weights(W0)
        run(straight, 0, 3)
        first = make()
        first.load_weights(W0)
        run(first, 0, 2)
        ck = {"W": [w.clone() for w in first.weights], "state": first.state_dict()}
        resumed = make()
        resumed.load_weights(ck["W"])
        resumed.load_state_dict(ck["state"])
        run(resumed, 2, 3)
        same = all(torch.equal(a, b) for a, b in zip(straight.weights, resumed.weights)) and \
            all(torch.equal(straight.momenta[i], resumed.momenta[i]) for i in straight.momenta)
        q.put((rank, same))
    finally:
        dist.destroy_process_group()


def test_sharded_checkpoint_resume_equals_straight_run():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_resume_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(same for _, same in out)


def test_state_dict_rejects_another_layout():
    import torch
    from spectral_optimizer_state_b200.sharded import ShardedMuon
    opt = ShardedMuon(SHAPES, dtype=torch.float64, device="cpu", local_step=_oracle_step,
                      state_dtype=torch.float64, **HP)
    st = opt.state_dict()
    other = ShardedMuon(SHAPES[:-1], dtype=torch.float64, device="cpu", local_step=_oracle_step,
                        state_dtype=torch.float64, **HP)
    with pytest.raises(ValueError):
        other.load_state_dict(st)
    opt.load_state_dict(st)  # round trip on the same layout
