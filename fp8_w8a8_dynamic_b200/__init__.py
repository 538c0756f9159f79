"""B200-native (sm_100a) FP8_DYNAMIC quantized Linear.

``mfp8`` is the Python binding of the C ABI in include/mfp8.h (libmfp8.so);
``workloads`` draws the seeded synthetic inputs.  Importing the package does
not load the CUDA library; the first call into ``mfp8`` does, and raises if
it has not been built.
"""
from . import workloads  # noqa: F401

__all__ = ["mfp8", "workloads", "build"]
