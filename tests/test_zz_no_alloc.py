"""The allocation-free momentum / norm entry point (for callers that cannot
call cudaMalloc) against the same pass inside muon_step, and against the fp64
oracle's momentum and look-ahead norm.

Collected last on purpose: the GPU test also passes after every other test
has used the library in the same process.
"""
import ctypes

import numpy as np
import pytest

import oracle
from synthetic import gaussian_spike, rng_for, round_bf16


def _lib():
    from spectral_optimizer_state_b200 import load_library
    from spectral_optimizer_state_b200.build import build
    build()
    return load_library()


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    # rejected on the host before any CUDA call: 24 x (4096 x 8192) needs 98304 partial sums
    lib = _lib()
    ptrs = (ctypes.c_void_p * 24)(*([1] * 24))
    st = lib.muon_momentum_norm_noalloc(ptrs, ptrs, ctypes.c_void_p(1), 24, 4096, 8192, 0, 0.95, 1, None)
    assert st == 2  # MUON_ERR_UNSUPPORTED_SHAPE
    assert lib.muon_momentum_norm_noalloc(None, None, None, 1, 8, 8, 0, 0.95, 1, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("shape,dtype", [((200, 328), "bf16"), ((3352, 768), "bf16"), ((257, 700), "f32")])
def test_noalloc_matches_muon_step_two_calls(shape, dtype):
    import torch
    from spectral_optimizer_state_b200 import Muon, momentum_norm_noalloc
    batch, beta = 3, 0.95
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    mu = Muon(0)
    W = [torch.zeros(shape, dtype=tdt, device="cuda") for _ in range(batch)]
    M_ref = [torch.zeros(shape, dtype=torch.float32, device="cuda") for _ in range(batch)]
    M_new = [torch.zeros(shape, dtype=torch.float32, device="cuda") for _ in range(batch)]
    nu = torch.full((batch,), -1.0, dtype=torch.float32, device="cuda")
    M_or = [np.zeros(shape) for _ in range(batch)]
    for call in range(2):
        G = []
        for l in range(batch):
            g = gaussian_spike(rng_for(700 + call, l), *shape).astype(np.float32)
            g = round_bf16(g) if dtype == "bf16" else g
            G.append(torch.from_numpy(g).to(tdt).cuda())
        mu.step(W, G, M_ref, lr=0.02, beta=beta, weight_decay=0.1, eps=1e-7)
        ref_nu = mu.norms()
        momentum_norm_noalloc(G, M_new, nu, beta=beta, nesterov=True)
        torch.cuda.synchronize()
        for l in range(batch):
            a = M_new[l].double().cpu().numpy()
            b = M_ref[l].double().cpu().numpy()
            assert np.linalg.norm(a - b) <= 1e-6 * np.linalg.norm(b)
            assert abs(float(nu[l]) - ref_nu[l]) <= 1e-5 * ref_nu[l]
            # and against the fp64 oracle's momentum and look-ahead norm
            g64 = G[l].double().cpu().numpy()
            M_or[l] = oracle.momentum_update(M_or[l], g64, beta)
            nu_or = oracle.frobenius_norm(oracle.nesterov_lookahead(g64, M_or[l], beta))
            assert np.linalg.norm(a - M_or[l]) <= 1e-6 * np.linalg.norm(M_or[l])
            assert abs(float(nu[l]) - nu_or) <= 1e-5 * nu_or
    mu.close()
