"""fp64 CPU oracle of the Muon step (test infrastructure only; see muon_oracle)."""
from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import (DEFAULT_COEFFS, DEFAULT_MOMENTUM, DEFAULT_NS_STEPS, DEFAULT_RMS_SCALE,
                          StepResult, apply_update, frobenius_normalise, gram, momentum, muon_step,
                          nesterov_input, newton_schulz, ns_iterate, poly, update_rms, update_scale)
