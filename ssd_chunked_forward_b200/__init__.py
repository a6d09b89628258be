"""B200-native chunked SSD forward.

The compute path is the C-ABI library ``libssd.so`` (CUDA kernels for
sm_100a, declared in ``include/ssd.h``); ``ssd_chunked_forward_b200.ssd``
is a thin ctypes binding over it.  Importing this package loads nothing:
the library is opened on first use and a missing library is an error, never
a silent fallback.
"""

__all__ = ["ssd", "workloads"]
