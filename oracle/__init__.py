"""fp64 CPU oracle of the Muon step.  TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check in __graft_entry__.py and bench.py's CPU-baseline /
reference leg may import anything here.  The CUDA library neither imports nor
links it, and it shares no code with the library.
"""
from .muon_oracle import (NS_COEFFS, NS_STEPS, DEFAULT_EPS, SCALE_NONE, SCALE_MATCH_RMS,
                          SCALE_CUSTOM, momentum_accumulate, nesterov_direction, orient,
                          frobenius_normalize, gram, poly_matrix, ns_update, ns_iteration,
                          newton_schulz, shape_scale, apply_update, muon_step, muon_steps, qk_clip)
from .jacobi_svd import jacobi_svd

__all__ = ["NS_COEFFS", "NS_STEPS", "DEFAULT_EPS", "SCALE_NONE", "SCALE_MATCH_RMS", "SCALE_CUSTOM",
           "momentum_accumulate", "nesterov_direction", "orient", "frobenius_normalize", "gram",
           "poly_matrix", "ns_update", "ns_iteration", "newton_schulz", "shape_scale",
           "apply_update", "muon_step", "muon_steps", "qk_clip", "jacobi_svd"]
