"""sp24: B200-native 2:4 semi-structured sparse GEMM (sm_100a).

The compute path lives in the CUDA shared library ``libsp24.so`` (sources in
``csrc/``), reached through the C ABI declared in ``include/sp24.h``.  The
Python module ``sp24`` only marshals arguments into that ABI; it has no
fallback and raises if the library is missing.
"""
__all__ = ["sp24", "inputs"]
