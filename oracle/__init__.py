"""fp64 CPU oracle for the KDA recurrence and its Gated DeltaNet special case.
Test infrastructure only: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product package."""
from .kda_oracle import (build, gdn_backward, gdn_decode_step, gdn_recurrence, kda_backward,
                         kda_decode_step, kda_layer,
                         kda_recurrence, kimi_log_alpha, l2_normalize, max_threads,
                         rms_norm_gate, sigmoid, softplus)

__all__ = ["build", "kda_recurrence", "kda_backward", "gdn_backward", "kda_decode_step", "gdn_recurrence", "gdn_decode_step",
           "kda_layer", "l2_normalize", "softplus", "sigmoid", "kimi_log_alpha", "rms_norm_gate",
           "max_threads"]
