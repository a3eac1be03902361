"""FP8 training GEMMs with dynamic tensorwise scaling for B200 (sm_100a).

The compute path is libfp8lm.so (C ABI in include/lm_fp8.h); ``_lib`` is its
ctypes binding and ``api`` adds PyTorch-allocated buffers around it.  Both
import the library eagerly and fail if it is not built.  ``synthetic`` holds
the seeded input generators and needs no GPU.
"""
__all__ = ["api", "synthetic"]
