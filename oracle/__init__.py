"""fp64 CPU oracle for the RainFusion2.0 block-sparse attention hot path.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU-baseline
leg import it.  It shares no code with the CUDA library.
"""
from .rf2_oracle import *  # noqa: F401,F403
from .rf2_oracle import Geom, Selection  # noqa: F401
