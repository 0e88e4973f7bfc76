"""B200-native (sm_100a) MoE expert layer.

The compute path is the CUDA library ``libmoe_b200.so`` built from ``csrc/`` and
reached through its C ABI (``include/moe.h``); ``moe`` is a thin ctypes binding
(argument marshalling only).  ``inputs`` holds the seeded synthetic workloads.
Importing this package loads nothing; ``moe`` loads the library on first use
and raises if it is missing.
"""
