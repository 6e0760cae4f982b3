"""Thin ctypes binding of libw4a16.so (C ABI in include/w4a16.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Functions carry the C names; pointer arguments accept torch tensors
(their ``data_ptr()``), numpy arrays (host pointers) or plain integers, and
``stream`` accepts a torch.cuda.Stream, a raw handle or None (the current
torch stream of the current device).  If the shared library is missing the
first call raises: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libw4a16.so")

FMT_INT4_G128 = 0
FMT_NVFP4_G16 = 1
FMT_FP8_E4M3 = 2
FMT_NVFP4_BS = 3
FMTS = {"int4": FMT_INT4_G128, "nvfp4": FMT_NVFP4_G16, "fp8": FMT_FP8_E4M3, "nvfp4_bs": FMT_NVFP4_BS}

OK = 0
ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_DEVICE, ERR_CUDA, ERR_TIMEOUT, ERR_NOMEM = -1, -2, -3, -4, -5, -6, -7
ERR_SCRATCH = -8
PATH_AUTO, PATH_GEMV, PATH_TC, PATH_BS = 0, 1, 2, 3
MAX_M = 8192

_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_SIGS = {
    "w4a16_packed_weight_bytes": (ctypes.c_size_t, [_i, _i, _i]),
    "w4a16_packed_scale_bytes": (ctypes.c_size_t, [_i, _i, _i]),
    "w4a16_pack_host": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp]),
    "w4a16_unpack_host": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp]),
    "w4a16_pack": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_dequant": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_ex": (_i, [_i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_path": (_i, [_i, _i, _i, _i]),
    "w4a16_gemm_gate_up_silu": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_gate_up_silu_ex": (_i, [_i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_noalloc": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_quantize_act_nvfp4": (_i, [_i, _i, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_w4a4": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_w4a4_ex": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_gemm_w4a4_bs": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_device_status": (_i, [_vp]),
    "w4a16_selftest_wait_timeout": (_i, [_vp]),
    "w4a16_plan": (_i, [_i, _i, _i, _i, _i, _i, _i, _vp, _i]),
    "w4a16_status_string": (ctypes.c_char_p, [_i]),
    "w4a16_version": (_i, []),
}


class W4A16Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}" if what else status_string(status))


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with __graft_entry__.build()")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if hasattr(a, "ctypes"):
        return a.ctypes.data
    raise TypeError(f"cannot pass {type(a)} as a pointer")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def status_string(status: int) -> str:
    return lib().w4a16_status_string(status).decode()


def check(status: int, what: str = "") -> None:
    if status != OK:
        raise W4A16Error(status, what)


def w4a16_packed_weight_bytes(fmt, N, K):
    return lib().w4a16_packed_weight_bytes(fmt, N, K)


def w4a16_packed_scale_bytes(fmt, N, K):
    return lib().w4a16_packed_scale_bytes(fmt, N, K)


def w4a16_pack_host(fmt, N, K, codes, scales, packed_w, packed_scales):
    return lib().w4a16_pack_host(fmt, N, K, _ptr(codes), _ptr(scales), _ptr(packed_w),
                                 _ptr(packed_scales))


def w4a16_unpack_host(fmt, N, K, packed_w, packed_scales, codes, scales):
    return lib().w4a16_unpack_host(fmt, N, K, _ptr(packed_w), _ptr(packed_scales), _ptr(codes),
                                   _ptr(scales))


def w4a16_pack(fmt, N, K, codes, scales, packed_w, packed_scales, stream=None):
    return lib().w4a16_pack(fmt, N, K, _ptr(codes), _ptr(scales), _ptr(packed_w),
                            _ptr(packed_scales), _stream(stream))


def w4a16_dequant(fmt, N, K, packed_w, packed_scales, global_scale, w_bf16, stream=None):
    return lib().w4a16_dequant(fmt, N, K, _ptr(packed_w), _ptr(packed_scales), _ptr(global_scale),
                               _ptr(w_bf16), _stream(stream))


def w4a16_gemm(fmt, M, N, K, x, packed_w, packed_scales, global_scale, y, stream=None):
    return lib().w4a16_gemm(fmt, M, N, K, _ptr(x), _ptr(packed_w), _ptr(packed_scales),
                            _ptr(global_scale), _ptr(y), _stream(stream))


def w4a16_gemm_ex(path, fmt, M, N, K, x, packed_w, packed_scales, global_scale, y, stream=None):
    return lib().w4a16_gemm_ex(path, fmt, M, N, K, _ptr(x), _ptr(packed_w), _ptr(packed_scales),
                               _ptr(global_scale), _ptr(y), _stream(stream))


def w4a16_gemm_noalloc(fmt, M, N, K, x, packed_w, packed_scales, global_scale, y, stream=None):
    return lib().w4a16_gemm_noalloc(fmt, M, N, K, _ptr(x), _ptr(packed_w), _ptr(packed_scales),
                                    _ptr(global_scale), _ptr(y), _stream(stream))


def w4a16_gemm_gate_up_silu(fmt, M, I, K, x, packed_w, packed_scales, global_scale, h,
                            stream=None):
    return lib().w4a16_gemm_gate_up_silu(fmt, M, I, K, _ptr(x), _ptr(packed_w),
                                         _ptr(packed_scales), _ptr(global_scale), _ptr(h),
                                         _stream(stream))


def w4a16_gemm_gate_up_silu_ex(path, fmt, M, I, K, x, packed_w, packed_scales, global_scale, h,
                               stream=None):
    return lib().w4a16_gemm_gate_up_silu_ex(path, fmt, M, I, K, _ptr(x), _ptr(packed_w),
                                            _ptr(packed_scales), _ptr(global_scale), _ptr(h),
                                            _stream(stream))


def w4a16_quantize_act_nvfp4(M, K, x, codes, scales, g_x, stream=None):
    return lib().w4a16_quantize_act_nvfp4(M, K, _ptr(x), _ptr(codes), _ptr(scales), _ptr(g_x),
                                          _stream(stream))


def w4a16_gemm_w4a4(M, N, K, x, packed_w, packed_scales, global_scale_w, y, stream=None):
    return lib().w4a16_gemm_w4a4(M, N, K, _ptr(x), _ptr(packed_w), _ptr(packed_scales),
                                 _ptr(global_scale_w), _ptr(y), _stream(stream))


def w4a16_gemm_w4a4_ex(path, M, N, K, x, packed_w, packed_scales, global_scale_w, y, stream=None):
    return lib().w4a16_gemm_w4a4_ex(path, M, N, K, _ptr(x), _ptr(packed_w), _ptr(packed_scales),
                                    _ptr(global_scale_w), _ptr(y), _stream(stream))


def w4a16_gemm_path(fmt, M, N, K):
    return lib().w4a16_gemm_path(fmt, M, N, K)


def w4a16_device_status(stream=None):
    return lib().w4a16_device_status(_stream(stream))


def w4a16_plan(path, fmt, M, N, K, fuse=0, num_sms=148):
    """(status or path, the nine plan fields) for a shape, computed on the host."""
    import numpy as np
    out = np.zeros(9, dtype=np.int32)
    r = lib().w4a16_plan(path, fmt, M, N, K, fuse, num_sms, out.ctypes.data, 9)
    return r, [int(v) for v in out]


def w4a16_selftest_wait_timeout(stream=None):
    return lib().w4a16_selftest_wait_timeout(_stream(stream))


def w4a16_version():
    return lib().w4a16_version()


# ---------------------------------------------------------------- torch-level conveniences
# (allocation and marshalling around the calls above)


def w4a16_gemm_w4a4_bs(M, N, K, x, packed_w, packed_sf, global_scale_w, y, stream=None):
    return lib().w4a16_gemm_w4a4_bs(M, N, K, _ptr(x), _ptr(packed_w), _ptr(packed_sf),
                                    _ptr(global_scale_w), _ptr(y), _stream(stream))


def pack_on_device(fmt: str, N: int, K: int, codes, scales, stream=None):
    """Pack logical device tensors; returns (packed_w, packed_scales) uint8 CUDA tensors."""
    import torch
    f = FMTS[fmt]
    w = torch.empty(w4a16_packed_weight_bytes(f, N, K), dtype=torch.uint8, device=codes.device)
    s = torch.empty(w4a16_packed_scale_bytes(f, N, K), dtype=torch.uint8, device=codes.device)
    check(w4a16_pack(f, N, K, codes, scales, w, s, stream), "w4a16_pack")
    return w, s


def gemm(fmt: str, x, packed_w, packed_scales, N: int, global_scale=None, y=None, path=PATH_AUTO,
         stream=None):
    """y = x . W_deq^T for a BF16 CUDA tensor x [M][K]; returns y (BF16 [M][N])."""
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(w4a16_gemm_ex(path, FMTS[fmt], M, N, K, x, packed_w, packed_scales, global_scale, y,
                        stream), "w4a16_gemm")
    return y


def gate_up_silu(fmt: str, x, packed_w, packed_scales, I: int, global_scale=None, h=None,
                 path=PATH_AUTO, stream=None):
    """h = SiLU(x . W_gate^T) * (x . W_up^T) for a BF16 CUDA tensor x [M][K] and
    the packed [2I][K] gate/up weight; returns h (BF16 [M][I])."""
    import torch
    M, K = x.shape
    if h is None:
        h = torch.empty((M, I), dtype=torch.bfloat16, device=x.device)
    check(w4a16_gemm_gate_up_silu_ex(path, FMTS[fmt], M, I, K, x, packed_w, packed_scales,
                                     global_scale, h, stream), "w4a16_gemm_gate_up_silu")
    return h


def quantize_act_nvfp4(x, stream=None):
    """NVFP4 activation quantiser on a BF16 CUDA tensor x [M][K]: returns
    (codes uint8 [M][K], E4M3 scales uint8 [M][K/16], g_x fp32 [1])."""
    import torch
    M, K = x.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    scales = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
    g_x = torch.empty(1, dtype=torch.float32, device=x.device)
    check(w4a16_quantize_act_nvfp4(M, K, x, codes, scales, g_x, stream), "w4a16_quantize_act_nvfp4")
    return codes, scales, g_x


def gemm_w4a4(x, packed_w, packed_scales, N: int, global_scale_w, y=None, path=PATH_AUTO,
              stream=None):
    """W4A4 NVFP4 matmul of a BF16 CUDA tensor x [M][K]; returns y (BF16 [M][N])."""
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(w4a16_gemm_w4a4_ex(path, M, N, K, x, packed_w, packed_scales, global_scale_w, y, stream),
          "w4a16_gemm_w4a4")
    return y


def gemm_w4a4_bs(x, packed_w, packed_sf, N: int, global_scale_w, y=None, stream=None):
    """W4A4 NVFP4 matmul on the block-scaled tensor cores (weights packed with
    format "nvfp4_bs"); returns y (BF16 [M][N])."""
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(w4a16_gemm_w4a4_bs(M, N, K, x, packed_w, packed_sf, global_scale_w, y, stream),
          "w4a16_gemm_w4a4_bs")
    return y


def dequant(fmt: str, N: int, K: int, packed_w, packed_scales, global_scale=None, out=None,
            stream=None):
    import torch
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=packed_w.device)
    check(w4a16_dequant(FMTS[fmt], N, K, packed_w, packed_scales, global_scale, out, stream),
          "w4a16_dequant")
    return out
