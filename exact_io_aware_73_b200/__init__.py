"""B200-native exact, IO-aware attention forward (sm_100a).

The compute lives in ``libattn_b200.so`` (hand-written CUDA for sm_100a behind
a C ABI declared in ``include/attn_b200.h``).  This package is the thin
Python binding over that library (argument marshalling only) plus the seeded
synthetic input recipe in ``workloads``.
"""
