"""B200-native HSTU layer: CUDA kernels for sm_100a behind a C-ABI library.

Import `hstu_sequential_transducer_02_b200.binding` for the library calls; it
loads `libhstu.so` from this directory and raises if it is missing.
"""
__all__ = ["binding", "workload"]
