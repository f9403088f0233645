"""paged_block_quantized_b200: decode-phase PagedAttention over a block-pooled, group-wise
quantized KV cache, as hand-written sm_100a CUDA kernels behind a C ABI (include/pkv.h).

Submodules
  pkv        ctypes binding of libpkv.so (same entry-point names as the C header). Importing it
             loads the CUDA library and raises if it has not been built.
  workloads  seeded synthetic inputs (shapes, lengths, block assignment, token values); holds no
             quantization or attention arithmetic.
  build      compiles libpkv.so for sm_100a with nvcc.

Importing the package itself loads nothing.
"""

__all__ = ["pkv", "workloads", "build"]
