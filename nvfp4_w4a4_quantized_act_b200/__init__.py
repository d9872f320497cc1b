"""B200-native NVFP4 W4A4 linear layer: on-the-fly activation quantization
and a tcgen05 block-scaled FP4 GEMM with a per-module global-scale epilogue.

The compute lives in the CUDA shared library ``libnvfp4.so`` (built from
``csrc/``); ``ops`` is a thin ctypes binding over its C ABI.  Importing the
package does not load the library; the first call does, and fails loudly if
the library or a CUDA device is missing.
"""
__all__ = ["ops", "workloads"]
