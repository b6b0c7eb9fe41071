"""frt: the fused static-FP8 attention-input chain on sm_100a (B200).

Subpackages/modules:
  frt      ctypes binding of libfrt.so (the C ABI of include/frt.h)
  runtime  device-buffer plumbing around the binding (torch memory/streams)
  synth    seeded synthetic inputs of the five workloads
  build    nvcc build of libfrt.so

Importing this package loads nothing; ``fp8_transformer_block_b200.frt``
loads the CUDA library and raises if it is missing.
"""

__all__ = ["frt", "runtime", "synth", "build"]
