"""B200-native (sm_100a) hybrid Top-k+Top-p block-sparse attention.

The compute path lives in ``libspa2.so`` (CUDA kernels behind a C ABI declared
in ``include/spa2.h``); ``binding`` wraps its entry points with ctypes. This
package import is light: the library is loaded on first use of ``binding``.
"""

__version__ = "0.1.0"
