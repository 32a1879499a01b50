"""B200-native rotated W4A4 linear layer (Omega-QVLA style).

The compute path lives in the shared library built from ``csrc/`` and is
reached through :mod:`w4a4_post_quantization_zigzag_b200.qvla` (a ctypes
binding).  Importing this package does not load the library; importing the
binding does, and fails loudly if it has not been built.
"""
__all__ = ["inputs", "qvla"]
