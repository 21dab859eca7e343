"""B200-native (sm_100a) NVFP4 quantised linear layer: fprop, dgrad and wgrad as
quantise-then-GEMM, behind the C ABI of include/nvfp4.h.

The compute runs in libnvfp4.so (CUDA, built in-tree by build.py); this package
only marshals torch tensors into that ABI.  Importing the package does not load
the library: the first call does, and fails loudly if it is missing.
"""

__all__ = ["api", "synthetic"]
