"""Failure detection without a GPU fault: a dropped completion signal ends in the bounded waits
(MUON_ERR_TIMEOUT), the weights are left as they were, and the context keeps working (needs a B200)."""
import os
import time

import numpy as np
import pytest

import oracle
from synthetic import gaussian_spike, group_weights, rng_for, round_bf16
from tests.gpu_common import to_device

pytestmark = pytest.mark.gpu

SHAPES = [(200, 328), (328, 200)]
COUNTS = [3, 2]
HP = dict(lr=0.02, beta=0.95, weight_decay=0.1, eps=1e-7, nesterov=True)


def _grads(step):
    return [[to_device(round_bf16(gaussian_spike(rng_for(950 + 10 * step + i, l), *SHAPES[i])), "bf16")
             for l in range(COUNTS[i])] for i in range(2)]


def test_dropped_signal_times_out_leaves_weights_and_context_recovers():
    import torch
    from spectral_optimizer_state_b200 import Muon
    os.environ["MUON_TEST_DROP_SIGNAL"] = "1"
    try:
        m = Muon(0)
    finally:
        del os.environ["MUON_TEST_DROP_SIGNAL"]
    m.set_coeffs([oracle.QUINTIC] * 5)
    W = [[to_device(w, "bf16") for w in group_weights(9, i, COUNTS[i], *SHAPES[i])] for i in range(2)]
    W0 = [[w.clone() for w in ws] for ws in W]
    M = [[torch.zeros(SHAPES[i], device="cuda") for _ in range(COUNTS[i])] for i in range(2)]
    t0 = time.time()
    m.step_groups([(W[i], _grads(0)[i], M[i]) for i in range(2)], **HP)
    st, flags = m.status()
    elapsed = time.time() - t0
    assert st == 6  # MUON_ERR_TIMEOUT
    assert elapsed < 30.0
    assert flags == [0] * sum(COUNTS)  # the norms were fine; the failure was the schedule's
    for ws, w0s in zip(W, W0):
        for w, w0 in zip(ws, w0s):
            assert torch.equal(w, w0)  # nothing applied from an incomplete iterate

    # the same context steps normally afterwards, exactly like a fresh one from the same state
    Wb = [[w.clone() for w in ws] for ws in W]
    Mb = [[x.clone() for x in ms] for ms in M]
    G1 = _grads(1)
    m.step_groups([(W[i], G1[i], M[i]) for i in range(2)], **HP)
    assert m.status()[0] == 0
    with Muon(0) as fresh:
        fresh.set_coeffs([oracle.QUINTIC] * 5)
        fresh.step_groups([(Wb[i], G1[i], Mb[i]) for i in range(2)], **HP)
        assert fresh.status()[0] == 0
    for i in range(2):
        for a, b, ma, mb in zip(W[i], Wb[i], M[i], Mb[i]):
            assert torch.equal(a, b) and torch.equal(ma, mb)
    m.close()
