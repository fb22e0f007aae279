"""fp64 CPU oracle of the Muon step (test infrastructure only).

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The library never does.
"""

from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import (NS_A, NS_B, NS_C, NS_EPS, adamw_step, apply_update,  # noqa: F401
                          muon_step, nesterov_momentum, newton_muon_step,
                          newton_schulz, quintic_scalar, right_precondition,
                          second_moment, shape_scale, spd_inverse)
