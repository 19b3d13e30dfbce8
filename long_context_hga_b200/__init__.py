"""HGA routed attention on B200: libhga.so (sm_100a CUDA kernels behind a C
ABI, see include/hga.h) and its ctypes binding `long_context_hga_b200.hga`.

The binding is imported lazily so that `long_context_hga_b200.build` works
before the library exists; importing `.hga` without a built libhga.so raises.
"""
import importlib

__all__ = ["hga", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
