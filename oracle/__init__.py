"""fp64 CPU oracle for the KDA recurrence and its Gated DeltaNet special case.
Test infrastructure only: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product package."""
from .kda_oracle import (build, gdn_decode_step, gdn_recurrence, kda_decode_step,
                         kda_recurrence, max_threads)

__all__ = ["build", "kda_recurrence", "kda_decode_step", "gdn_recurrence", "gdn_decode_step",
           "max_threads"]
