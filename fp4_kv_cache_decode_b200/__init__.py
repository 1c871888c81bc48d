"""B200-native CSA2 step over an FP4 KV cache.

The computation lives in ``lib/libcsa2.so`` (hand-written sm_100a CUDA kernels
behind the C ABI of ``include/csa2.h``); :mod:`.csa2` is its thin ctypes
binding.  Importing the package does not load the library; the first call does,
and fails loudly if it has not been built.
"""

__version__ = "0.1.0"
