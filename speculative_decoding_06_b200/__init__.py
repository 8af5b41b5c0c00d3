"""B200 (sm_100a) tree verification for EAGLE-3 speculative decoding.

The product is libspec.so (C ABI in include/spec.h); `spec` is its ctypes
binding and `engine.SpecEngine` a thin wrapper that supplies device memory and
the stream from PyTorch.
"""

from . import spec  # noqa: F401
