"""CPU oracle for the online W4A4 rotated linear layer (test infrastructure).

This package is test infrastructure.  Only the tests, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
The CUDA library never calls it and shares no code with it.
"""
from .qr_oracle import *  # noqa: F401,F403
