"""B200-native 4-bit-Muon-GRASP optimizer step.

The compute lives in ``libgmuon.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/gmuon.h``); ``gmuon`` is its thin ctypes binding.
``workloads`` draws seeded synthetic inputs and ``flops`` counts algorithmic
work for reporting.
"""

__all__ = ["gmuon", "workloads", "flops"]
