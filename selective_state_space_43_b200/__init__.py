"""B200-native Mamba-2 selective-SSM layer core (SSD prefill + decode).

The arithmetic runs in the CUDA library ``libssd_b200.so`` (sm_100a) behind a
C ABI declared in ``include/ssd.h``; :mod:`.ops` is a thin ctypes binding that
passes device pointers and the current stream.  Importing this package does
not load the library; the first op call does, and raises if it is missing.
"""
from .synth import Dims, WORKLOADS  # noqa: F401

__all__ = ["Dims", "WORKLOADS"]
