"""SVDQuant W4A4 + low-rank linear layer for B200 (sm_100a).

The compute lives in ``libsvdq.so`` (CUDA kernels behind the C ABI declared in
``include/svdq.h``); this package is its ctypes binding.
"""

from .binding import *  # noqa: F401,F403
from .binding import (  # noqa: F401
    EXPORTED,
    LIB_PATH,
    SvdqError,
    Weights,
    act_buffers,
    linear,
)
