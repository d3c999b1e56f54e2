"""fp64 CPU oracle for RIB windowed attention and its convolutional local
attention gate.

Test infrastructure: only tests/, the package smoke check and the benchmark's
CPU-baseline leg use it.  The CUDA library never imports or links it.
"""
from .rib_oracle import *  # noqa: F401,F403
from .rib_oracle import __all__ as _rib_all
from .cla_oracle import *  # noqa: F401,F403
from .cla_oracle import __all__ as _cla_all

__all__ = list(_rib_all) + list(_cla_all)
