"""Oracle for the OLMo 3 hybrid sliding-window attention path (TEST INFRASTRUCTURE).

A plain, slow, fp64 CPU statement of what the GPU library computes.  Only the
test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it.  It shares no code with the CUDA path and never
imports the package ``hybrid_sliding_window_olmo3_b200``.
"""
from .olmo3_oracle import *  # noqa: F401,F403
from .olmo3_oracle import __all__  # noqa: F401
