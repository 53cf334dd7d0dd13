"""B200-native (sm_100a) KDA (Kimi Delta Attention) recurrence.

``kda`` is the binding of the C-ABI library libkda.so (built in-tree by
``gated_delta_rule_61_b200.build``); ``inputs`` holds the seeded synthetic
input recipe. Importing the package does not load the library; the first
call does, and raises if it is missing.
"""
from . import inputs  # noqa: F401
from .kda import KdaError, decode_step, device_status, prefill  # noqa: F401

__all__ = ["prefill", "decode_step", "device_status", "KdaError", "inputs"]
