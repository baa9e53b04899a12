"""B200-native sparse Mixture-of-Experts FFN forward.

The layer runs in hand-written sm_100a CUDA kernels behind a C-ABI library
(``libmoe.so``); ``binding`` is the thin ctypes layer over it and ``synth`` draws
seeded synthetic workloads. Importing the package does not load the library.
"""
__all__ = ["synth", "binding"]
