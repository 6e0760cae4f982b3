"""W4A16 weight-only 4-bit matmul for NVIDIA B200 (sm_100a).

The computation lives in ``libw4a16.so`` (CUDA, C ABI in ``include/w4a16.h``);
``w4a16`` is its thin ctypes binding.  Build with ``__graft_entry__.build()``.
"""

from .w4a16 import (  # noqa: F401
    FMT_INT4_G128,
    FMT_NVFP4_G16,
    PATH_AUTO,
    PATH_GEMV,
    PATH_TC,
    W4A16Error,
    check,
    dequant,
    gemm,
    lib,
    pack_on_device,
)
