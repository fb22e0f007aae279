"""Muon optimizer step for one NVIDIA B200 (sm_100a).

The compute path is the CUDA library libmuon_b200.so (C ABI in
include/muon.h); this package only marshals torch tensors into it.
"""

from .binding import (MUON_BF16, MUON_F32, SCALE_MODES, MuonContext, MuonError,  # noqa: F401
                      default_adamw_hparams, default_hparams, load_library)
