"""fp64 CPU oracle (test infrastructure only; see ``oracle.muon_oracle``)."""
from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import (  # noqa: F401
    CUBIC, GRAM, GRAM_STABILIZED, MODES, QUINTIC, STANDARD,
    apply_update, flops, flops_gram, flops_standard, flops_standard_iteration,
    frobenius_norm, frobenius_normalize, is_restart, momentum_update, muon_step, nesterov_blend,
    newton_schulz, ns_gram, ns_gram_stored, ns_standard, ns_standard_stored, orient, round_to,
    singular_value_map,
    unorient, update_scale,
)
