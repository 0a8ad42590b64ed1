"""B200-native gated nD FFT long convolution (HyenaND hot path).

The product is the C-ABI shared library libhyena_nd.so (include/hyena_nd.h),
built from csrc/ for sm_100a.  ``hyena_nd`` is its thin Python binding.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads", "hyena_nd"]
