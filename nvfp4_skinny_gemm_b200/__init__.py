"""nvfp4_skinny_gemm_b200: B200 (sm_100a) kernels for the tree-MTP verification step.

The compute lives in ``libnvfp4sk.so`` (CUDA C++, C ABI declared in
``include/nvfp4sk.h``).  ``lib`` is the thin ctypes binding with the same
entry-point names; ``step`` composes those calls into the 64-layer verify
step.  Importing this package does not load the library; the first call does,
and it raises if the library is missing -- there is no CPU fallback.
"""
__all__ = ["lib", "inputs"]
