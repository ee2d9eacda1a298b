"""Checkpoint / resume: the optimizer state is the caller's M (and W); saving it after 5 steps
and resuming in a new context for 5 more is bit-identical to 10 straight steps (needs a B200)."""
import io

import pytest

import oracle
from synthetic import MAMBA2_130M_IN_PROJ, MAMBA2_130M_OUT_PROJ, group_inputs, group_weights
from tests.gpu_common import to_device

pytestmark = pytest.mark.gpu

SHAPES = [MAMBA2_130M_OUT_PROJ, MAMBA2_130M_IN_PROJ]
COUNT = 4
HP = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True)


def _grads(step):
    return [[to_device(g, "bf16") for g in group_inputs(3, step, i, COUNT, *SHAPES[i])] for i in range(2)]


def _fresh_state():
    import torch
    W = [[to_device(w, "bf16") for w in group_weights(3, i, COUNT, *SHAPES[i])] for i in range(2)]
    M = [[torch.zeros(SHAPES[i], device="cuda") for _ in range(COUNT)] for i in range(2)]
    return W, M


def _steps(mu, W, M, first, last):
    for s in range(first, last):
        G = _grads(s)
        mu.step_groups([(W[i], G[i], M[i]) for i in range(2)], **HP)
    assert mu.status()[0] == 0


def test_save_after_five_resume_for_five_equals_ten_straight():
    import torch
    from spectral_optimizer_state_b200 import Muon
    Wa, Ma = _fresh_state()
    with Muon(0) as mu:
        mu.set_coeffs([oracle.QUINTIC] * 5)
        _steps(mu, Wa, Ma, 0, 10)
    Wb, Mb = _fresh_state()
    with Muon(0) as mu:
        mu.set_coeffs([oracle.QUINTIC] * 5)
        _steps(mu, Wb, Mb, 0, 5)
    buf = io.BytesIO()
    torch.save({"W": [[w.cpu() for w in ws] for ws in Wb], "M": [[m.cpu() for m in ms] for ms in Mb],
                "step": 5}, buf)
    del Wb, Mb
    torch.cuda.synchronize()
    buf.seek(0)
    ck = torch.load(buf)
    Wc = [[w.cuda() for w in ws] for ws in ck["W"]]
    Mc = [[m.cuda() for m in ms] for ms in ck["M"]]
    with Muon(0) as mu:
        mu.set_coeffs([oracle.QUINTIC] * 5)
        _steps(mu, Wc, Mc, ck["step"], 10)
    for i in range(2):
        for a, c, ma, mc in zip(Wa[i], Wc[i], Ma[i], Mc[i]):
            assert torch.equal(a, c) and torch.equal(ma, mc)
