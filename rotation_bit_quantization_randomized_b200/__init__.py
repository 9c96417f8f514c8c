"""QuaRot online rotation + INT4 inference hot path for NVIDIA B200 (sm_100a).

The compute lives in libquarot.so (hand-written CUDA, C ABI declared in
include/quarot.h).  `binding` is a thin ctypes layer with the same entry-point
names; `synth` generates the seeded synthetic inputs.  Importing the package
does not load the library; importing `binding` does, and raises if the library
is missing -- there is no CPU fallback.
"""
import importlib

__all__ = ["binding", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
