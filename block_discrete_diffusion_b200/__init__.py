"""B200-native (sm_100a) block-diffusion canvas decoder.

The computation lives in libdg.so (hand-written CUDA for sm_100a behind the C ABI of include/dg.h);
``dg`` is its ctypes binding.  Importing this package does not load the library; the first call
through ``dg`` does, and fails loudly if the library has not been built.
"""
from . import dg  # noqa: F401

__all__ = ["dg"]
