"""B200-native fused speculative verify-and-distill (AdaFlash hot path).

The compute path is the CUDA library ``libsvd.so`` (built from ``csrc/``); this package only
marshals arguments to its C ABI.  Importing the package loads nothing: the library is opened on
first use, and every entry point raises if it is missing.
"""
__all__ = ["api", "synthetic"]
