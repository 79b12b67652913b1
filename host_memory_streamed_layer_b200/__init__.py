"""Host-memory-streamed layer training on B200 (sm_100a).

The compute path lives in the in-tree shared library `libmt.so` (CUDA kernels,
streaming engine and host optimizer, C ABI in include/mt.h and
include/mt_kernels.h). This package is a thin ctypes binding over it: argument
marshalling only. Importing `mt` raises if the library has not been built.
"""
