"""2-bit mixed-precision KV cache with fused decode attention for B200 (sm_100a).

The compute path is the C-ABI library ``libkvq.so`` (hand-written CUDA kernels);
this package only marshals arguments to it.  ``synthetic`` holds the seeded input
generators.  Importing the package does not load the library; the first call does,
and raises if the library is missing or the device cannot run it.
"""
from .binding import *  # noqa: F401,F403
from .binding import __all__ as _binding_all

__all__ = list(_binding_all)
