"""ADMM-Q layer solve on B200 (sm_100a).

The compute path is the C-ABI library `libadmmq.so` (hand-written CUDA for
sm_100a, declared in include/admmq.h); `admmq` is its thin ctypes binding.
The library is loaded on first use and a missing or unloadable library raises:
there is no CPU fallback.
"""
from . import workloads  # noqa: F401


def __getattr__(name):
    if name in ("admmq", "lib"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
