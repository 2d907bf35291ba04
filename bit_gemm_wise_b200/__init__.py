"""B200 (sm_100a) blockwise 4-bit weight quantization and the matmuls that consume it.

Modules:
  w4     -- ctypes binding of the C-ABI library ``libw4.so`` (argument marshalling only;
            every step of the path runs in the CUDA kernels of ``csrc/``).
  synth  -- seeded synthetic inputs (no quantization or matmul arithmetic).
  build  -- nvcc build of ``libw4.so`` for sm_100a.

Importing the package does not load the CUDA library; ``w4`` loads it on first use and
raises if it is missing.
"""
__all__ = ["w4", "synth", "build"]
