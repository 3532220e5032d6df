"""fp64 CPU oracle for the RainFusion2.0 block-sparse attention hot path (and, in
``oracle.rf1``, the RainFusion v1 mask generators that feed the same attention).

Test infrastructure: only the tests, the smoke check and the benchmark's CPU-baseline
leg import it.  It shares no code with the CUDA library.
"""
from .rf2_oracle import *  # noqa: F401,F403
from .rf2_oracle import Geom, Selection  # noqa: F401
from . import rf1_oracle as rf1  # noqa: F401  (RainFusion v1 mask generators)
from . import fp8_oracle as fp8  # noqa: F401  (e4m3 quantised attention)
