"""fp64 CPU oracle for CoWindow Attention -- test infrastructure only.

Only ``tests/``, the package smoke check and the bench's CPU-baseline leg may
import this package.  It never imports the CUDA library and shares no code
with it.
"""
from .oracle import *  # noqa: F401,F403
