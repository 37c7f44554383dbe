"""SVDQuant W4A4 + low-rank linear layer for B200 (sm_100a).

The compute lives in ``libsvdq.so`` (CUDA kernels behind the C ABI declared in
``include/svdq.h``); ``binding`` is its ctypes binding.  The binding is loaded
on first use of any name of this package, so that ``python -m
rank_outlier_gemm_b200.build`` can (re)build the library without loading it;
using the package without a built library raises ImportError.
"""

import importlib


def __getattr__(name):
    if name == "build":  # the build script never needs the built library
        return importlib.import_module(".build", __name__)
    binding = importlib.import_module(".binding", __name__)
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None


def __dir__():
    return sorted(set(globals()) | set(dir(importlib.import_module(".binding", __name__))))
