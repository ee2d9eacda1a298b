"""fp64 CPU oracle for the Muon weight update -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may import this package.  The product (spectral_optimizer_state_b200) never
imports it and shares no code with it; the only module both sides use is
`synthetic`, which draws seeded inputs and holds none of the method.

Every function follows, step by step and in float64, what the pages state
(Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
Muon orthogonalises each weight matrix's update with a Newton-Schulz
iteration, i.e. steepest descent under the spectral norm) together with the
plainest reading of the steps they leave open; each reading is listed in the
function that takes it.

Pins tie it to things other than itself.  tests/test_oracle_pins.py: the SVD
closed form U f_k(S) V^T of the iteration, the polar factor U V^T, the
fixed-point scaling of semi-orthogonal inputs, the singular-value band of the
polynomial, invariances, exact rational arithmetic on diagonal inputs, closed
forms of momentum and the decoupled update, and a scalar-loop transcription of
the whole step on tiny inputs.  tests/test_oracle_mutants.py: planted mistakes
are rejected.  tests/test_oracle_adamw.py: AdamW's first step, moment closed
forms, decay-only and scale cases, and the parameter selection.
tests/test_oracle_spectral.py: power iteration and the smallest singular value
against LAPACK and exact cases, and the cap's vanishing first-order growth.

Parity unpinned (parameters, not facts of the pages): the quintic coefficient
triple and the shape-scale convention.  Parity holds for whichever values are
passed.
"""
from .adamw_oracle import adamw_step, select_muon  # noqa: F401
from .spectral_oracle import (min_singular_shifted, muon_step_capped, power_iteration, spectral_cap,  # noqa: F401
                              stable_rank)
from .muon_oracle import (  # noqa: F401
    CUBIC, QUINTIC, SCALE_SQRT_RATIO, SCALE_NONE, SCALE_RMS_MATCH,
    momentum_update, nesterov_lookahead, frobenius_norm, normalize,
    wide_view, newton_schulz, orthogonalize, shape_scale, apply_update, muon_step,
)
