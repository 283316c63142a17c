"""SeedLM hot path on B200: on-the-fly reconstruction of LFSR-seeded weight
blocks fused with the GEMV / small-M GEMM that consumes them.

Submodules:
  inputs  -- seeded synthetic records and activations (NumPy only)
  seedlm  -- ctypes binding of the C-ABI library libseedlm.so (CUDA)
  build   -- nvcc build of libseedlm.so, in-tree
"""
__all__ = ["inputs", "seedlm", "build"]
