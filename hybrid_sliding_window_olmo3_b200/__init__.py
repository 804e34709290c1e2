"""OLMo 3 hybrid sliding-window attention on B200 (sm_100a).

The compute lives in ``libolmo3.so`` (hand-written CUDA behind a C ABI, see
``include/olmo3.h``); ``hybrid_sliding_window_olmo3_b200.olmo3`` is the thin
ctypes binding with the same names.  Importing this package does not load the
library; the first binding call does, and fails loudly if it is missing.
"""
__all__ = ["olmo3", "workloads"]
