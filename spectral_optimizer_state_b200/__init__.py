"""B200-native Muon weight update (libmuon): C-ABI library + thin ctypes binding.

See include/muon.h for the interface.  `Muon` is the context object; its
methods call libmuon.so directly.
"""
from .binding import (  # noqa: F401
    CUBIC, EXPORTS, FLAG_NONFINITE, MAX_BATCH, MAX_GROUPS, MAX_ITERS, MUON_BF16, MUON_F32, QUINTIC,
    SCALE_NONE, SCALE_RMS_MATCH, SCALE_SQRT_RATIO, AdamWGroup, Muon, MuonError, SpectralPlan, StepPlan, adamw_step,
    load_library, momentum_norm_noalloc,
)
from .optim import MuonAdamW, takes_muon, torch_optimizer  # noqa: F401,E402
