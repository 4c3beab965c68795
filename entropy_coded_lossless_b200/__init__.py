"""B200-native Shannonic entropy codec for INT8 ML tensors.

The codec (histogram → DP range selection → tANS tables → chunk-parallel encode / decode) runs
in hand-written sm_100a CUDA kernels behind the C ABI declared in include/shn.h. Submodules:
``shn`` is the thin ctypes binding over that library (import it explicitly) and ``inputs`` holds
the seeded synthetic workloads.
"""
