"""KDA (Kimi Delta Attention) operator for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libkda.so`` built from ``csrc/``;
``gated_delta_rule_69_b200.kda`` is the thin ctypes binding over it.
"""
from . import inputs  # noqa: F401
