"""B200-native Shannonic entropy codec for INT8 ML tensors.

The codec (histogram → DP range selection → tANS tables → chunk-parallel encode / decode) runs
in hand-written sm_100a CUDA kernels behind the C ABI declared in include/shn.h; ``shn`` is the
thin ctypes binding over that library and ``inputs`` holds the seeded synthetic workloads.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "shn"]


def __getattr__(name):
    if name == "shn":
        from . import shn as _shn

        return _shn
    raise AttributeError(name)
