"""B200 (sm_100a) MX block-scaled matrix multiply C = A * B^T.

Submodules:
  mxgemm  -- ctypes binding of libmxgemm.so (the C ABI in include/mxgemm.h)
  synth   -- seeded synthetic FP32 inputs of the benchmark workloads
  build   -- builds libmxgemm.so in-tree with nvcc (sm_100a)

The binding is imported on demand so that ``synth`` stays usable without the
compiled library.
"""

__all__ = ["mxgemm", "synth", "build"]
