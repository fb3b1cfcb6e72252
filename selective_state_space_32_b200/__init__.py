"""B200-native selective-scan (Mamba / S6) forward.

The compute path is a CUDA library for sm_100a (``csrc/``) behind a C ABI
(``include/sscan.h``); ``sscan`` is its thin ctypes binding.  ``workloads``
draws seeded synthetic inputs.  Importing the package loads nothing: the
native library is opened on first use and a missing build is an error.
"""
__all__ = ["workloads", "sscan"]
