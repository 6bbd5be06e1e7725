"""B200-native context-parallel attention hot path.

Ring attention (fp32 partial output + LSE merged with the LSE rule), the
Ulysses sequence<->head permutation (including uneven 'anything' splits),
kv_gather and unified ring x Ulysses attention, as hand-written sm_100a CUDA
kernels behind the C ABI declared in include/cpattn.h (libcpattn.so).

Importing this package does not load the native library; ``api`` does, and
fails loudly if it is missing.
"""
__all__ = ["inputs", "api"]
