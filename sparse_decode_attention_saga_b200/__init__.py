"""SAGA + Atop-N single-token decode attention for B200 (sm_100a).

The compute lives in ``libsaga.so`` (hand-written CUDA behind the C ABI in
include/saga.h); this package is its ctypes binding (``_lib``), a host-side
decode-loop driver (``decoder``), the seeded synthetic workloads
(``workload``) and the build script (``build``).  Importing the package does
not load the library; the first call does, and fails loudly if it is absent.
"""
from . import workload  # noqa: F401

__all__ = ["workload", "decoder", "_lib", "build"]


def __getattr__(name):
    if name in ("decoder", "_lib", "build"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    if name == "AtopNDecoder":
        from .decoder import AtopNDecoder
        return AtopNDecoder
    raise AttributeError(name)
