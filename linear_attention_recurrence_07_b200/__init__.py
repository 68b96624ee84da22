"""Gated DeltaNet token mixer for NVIDIA B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA behind a C ABI declared
in ``include/gdn.h``).  ``binding`` is a thin ctypes layer over it; ``inputs``
draws the seeded synthetic workloads.  The shared library is loaded on first
use and its absence is an error: there is no CPU fallback.
"""
__all__ = ["binding", "inputs"]


def __getattr__(name):
    if name in ("binding", "inputs"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    if name in ("gdn_chunk_fwd", "gdn_decode_step", "GdnError"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
