"""CPU oracle of WeDLM Streaming Parallel Decoding (fp64, numpy).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
benchmark's CPU-baseline leg, never by the CUDA library or its Python binding.
It shares no code with the CUDA path.  Every function is pinned by the
``-m "not gpu"`` tests in tests/test_oracle_*.py.
"""
from .wedlm_oracle import *  # noqa: F401,F403
from . import wedlm_oracle  # noqa: F401
