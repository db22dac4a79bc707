"""B200-native Gated DeltaNet (GDN) token mixer.

The compute lives in ``libgdn.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/gdn.h``).  :mod:`.gdn` is the thin ctypes binding with the
same entry-point names; :mod:`.inputs` draws the seeded synthetic workloads.
"""
__all__ = ["gdn", "inputs"]


def __getattr__(name):
    if name == "gdn":
        from . import gdn as _gdn
        return _gdn
    raise AttributeError(name)
