"""DSpark draft/verify round on one B200: CUDA kernels behind a C ABI, with a thin ctypes binding.

Importing the package does not load the CUDA library; `speculative_decoding_04_b200.dspark`
does, and raises if it is missing (there is no CPU fallback).
"""
