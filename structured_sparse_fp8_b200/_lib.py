"""ctypes loader for ``libsp24.so`` (the C ABI declared in ``include/sp24.h``).

Loading fails loudly when the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsp24.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "sp24.h")

SP24_OK = 0
SP24_ERR_NULL = -1
SP24_ERR_SHAPE = -2
SP24_ERR_ALIGN = -3
SP24_ERR_DTYPE = -4
SP24_ERR_CUDA = -5
SP24_ERR_WORKSPACE = -6
SP24_ERR_ARCH = -7
SP24_STATUS_NONFINITE = 1
SP24_STATUS_TIMEOUT = 2
DTYPE_E4M3 = 0
DTYPE_BF16 = 1
(OP_QUANTIZE, OP_PRUNE_COMPRESS, OP_SLIDE68_DECOMPOSE, OP_SLIDE68_LIFT, OP_GEMM, OP_GEMM_DENSE,
 OP_GEMM_PACKED, OP_QUANTIZE_GEMM_PACKED, OP_LIFT_GEMM_PACKED, OP_GEMM_FP4) = range(10)

_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t

SIGNATURES = {
    "sp24_prune_compress": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _sz, _p, _p]),
    "fp8_quantize_pertensor": (_i, [_p, _i64, _i64, _p, _p, _p, _sz, _p, _p]),
    "fp8_quantize_pertensor_static": (_i, [_p, _i64, _i64, _p, _p, _p, _p]),
    "slide68_decompose": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _sz, _p, _p]),
    "slide68_lift": (_i, [_p, _i, _i, _p, _p, _p, _sz, _p, _p]),
    "sp24_gemm": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _sz, _p, _p]),
    "fp8_gemm_dense": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _sz, _p, _p]),
    "sp24_pack_weights": (_i, [_p, _p, _i, _i, _p, _p]),
    "sp24_prune_compress_packed": (_i, [_p, _i, _i, _p, _p, _p, _sz, _p, _p]),
    "slide68_decompose_packed": (_i, [_p, _i, _i, _p, _p, _p, _sz, _p, _p]),
    "sp24_gemm_packed": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _sz, _p, _p]),
    "sp24_quantize_gemm_packed": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _sz, _p, _p]),
    "slide68_lift_gemm_packed": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _sz, _p, _p]),
    "fp8_quantize_pertoken": (_i, [_p, _i64, _i64, _p, _p, _p, _p]),
    "slide_decompose": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _sz, _p, _p]),
    "int8_quantize_pertensor": (_i, [_p, _i64, _i64, _p, _p, _p, _sz, _p, _p]),
    "sp24_prune_compress_int8": (_i, [_p, _i, _i, _p, _p, _p, _p, _sz, _p, _p]),
    "sp24_gemm_int8_packed": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _sz, _p, _p]),
    "fp4_quantize_pertensor": (_i, [_p, _i64, _i64, _p, _p, _p, _sz, _p, _p]),
    "sp24_prune_compress_fp4": (_i, [_p, _i, _i, _p, _p, _p, _p, _sz, _p, _p]),
    "sp24_gemm_fp4": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _sz, _p, _p]),
    "slide_lift": (_i, [_p, _i, _i, _i, _p, _p, _p, _sz, _p, _p]),
    "sp24_prune_compress_perchannel": (_i, [_p, _i, _i, _p, _p, _p, _p, _p]),
    "sp24_gemm_packed_scaled": (_i, [_p, _p, _i, _p, _p, _i, _p, _i, _i, _i, _p, _sz, _p, _p]),
    "sp24_workspace_size": (_sz, [_i, _i64, _i64, _i64, _i]),
    "sp24_status_str": (ctypes.c_char_p, [_i]),
    "sp24_last_cuda_error": (_i, []),
    "sp24_debug_e4m3_encode": (_i, [_p, _p, _i64, _p]),
    "sp24_version": (ctypes.c_char_p, []),
}

_LIB = None


def header_functions() -> list[str]:
    """Names of every function declared in include/sp24.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)


def load() -> ctypes.CDLL:
    """Load libsp24.so once and bind every exported function's signature."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m structured_sparse_fp8_b200.build` "
            "(there is no CPU or eager fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


class Sp24Error(RuntimeError):
    pass


def check(rc: int, what: str) -> None:
    if rc != SP24_OK:
        lib = load()
        msg = lib.sp24_status_str(rc).decode()
        if rc == SP24_ERR_CUDA:
            msg += f" (cudaError {lib.sp24_last_cuda_error()})"
        raise Sp24Error(f"{what} failed: {msg} [{rc}]")
