"""B200-native NVFP4 hot path: two-level quantization and block-scaled FP4
GEMM on sm_100a, behind the C ABI of libnvfp4.so (include/nvfp4.h).

``binding`` is the thin Python layer over that ABI; ``inputs`` draws the
seeded synthetic workloads.  Importing this package does not need a GPU;
calling an operation without the built library raises.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "binding"]


def __getattr__(name):
    if name == "binding":
        import importlib
        return importlib.import_module(__name__ + ".binding")
    raise AttributeError(name)
