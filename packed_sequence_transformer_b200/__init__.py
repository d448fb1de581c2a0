"""B200-native packed-sequence Transformer layer (jagged causal attention +
top-2 MoE) behind a C ABI (include/ptl.h, libptl.so).

  ptl        -- ctypes binding of the C ABI (torch tensors in, kernels run in libptl.so)
  synthetic  -- seeded synthetic workloads shaped like the README's packed batches
  build      -- in-tree nvcc build of libptl.so for sm_100a
"""
from . import synthetic  # noqa: F401

__all__ = ["ptl", "synthetic", "build"]
