"""CPU oracle for TurboQuant-style KV compression and compressed-cache decode attention.

TEST INFRASTRUCTURE ONLY. Only the test-suite, the smoke check in ``__graft_entry__`` and
the CPU-baseline leg of ``bench.py`` may import this package. The product path (the CUDA
library and its Python binding) never imports, links or executes anything here.
"""
from .tq_oracle import *  # noqa: F401,F403
