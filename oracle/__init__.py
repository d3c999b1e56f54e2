"""fp64 CPU oracle for RIB windowed attention.

Test infrastructure: only tests/, the package smoke check and the benchmark's
CPU-baseline leg use it.  The CUDA library never imports or links it.
"""
from .rib_oracle import *  # noqa: F401,F403
from .rib_oracle import __all__  # noqa: F401
