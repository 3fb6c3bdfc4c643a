"""ctypes view of libqlora_nf4.so (the C ABI in include/qlora_nf4.h).

Argument marshalling only.  Importing this module loads the shared library
and raises ImportError if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_INVALID_ARG = 1
QLORA_ERR_UNSUPPORTED = 2
QLORA_ERR_NONFINITE = 3
QLORA_ERR_BAD_PADDING = 4
QLORA_ERR_CUDA = 5
QLORA_ERR_TIMEOUT = 6
QLORA_DTYPE_BF16 = 0
QLORA_DTYPE_F32 = 1
ABI_VERSION = 2
NOALLOC_MAX_NUMEL = 1 << 26


class NF4StateC(C.Structure):
    """Mirror of ``qlora_nf4_state``."""
    _fields_ = [
        ("numel", C.c_int64),
        ("blocksize", C.c_int32),
        ("double_quant", C.c_int32),
        ("dq_blocksize", C.c_int32),
        ("codebook", C.c_int32),
        ("packed", C.c_void_p),
        ("absmax", C.c_void_p),
        ("code8", C.c_void_p),
        ("s2", C.c_void_p),
        ("offset", C.c_void_p),
    ]


# name -> (restype, argtypes): every symbol the header declares
_VP, _I64, _I32, _SZ, _F = C.c_void_p, C.c_int64, C.c_int32, C.c_size_t, C.c_float
_PS = C.POINTER(NF4StateC)
SIGNATURES = {
    "qlora_abi_version": (_I32, []),
    "qlora_status_str": (C.c_char_p, [_I32]),
    "qlora_last_cuda_error": (C.c_char_p, []),
    "qlora_nf4_n1": (_I64, [_I64]),
    "qlora_nf4_n2": (_I64, [_I64]),
    "qlora_status_sync": (_I32, [_VP, _VP, C.POINTER(C.c_int32)]),
    "qlora_status_clear": (_I32, [_VP, _VP]),
    "qlora_nf4_quantize_workspace_size": (_SZ, [_I64, _I32]),
    "qlora_nf4_quantize": (_I32, [_VP, _I32, _PS, _VP, _SZ, _VP, _VP]),
    "qlora_nf4_quantize_noalloc": (_I32, [_VP, _I32, _PS, _VP, _VP]),
    "qlora_nf4_quantize_shard_workspace_size": (_SZ, [_I64, _I64, _I64, _I32]),
    "qlora_nf4_quantize_shard_begin": (_I32, [_VP, _I32, _PS, _I64, _I64, _VP, _SZ, _VP, _VP]),
    "qlora_nf4_quantize_shard_end": (_I32, [_PS, _I64, _I64, _VP, _SZ, _VP, _VP]),
    "qlora_nf4_dequantize": (_I32, [_PS, _VP, _VP, _VP]),
    "qlora_linear_fwd_workspace_size": (_SZ, [_I64, _I64, _I64, _I32]),
    "qlora_linear_fwd": (_I32, [_I64, _I64, _I64, _I32, _VP, _PS, _VP, _VP, _F, _VP, _VP,
                                _VP, _SZ, _VP, _VP]),
    "qlora_linear_bwd_workspace_size": (_SZ, [_I64, _I64, _I64, _I32]),
    "qlora_linear_bwd": (_I32, [_I64, _I64, _I64, _I32, _VP, _VP, _VP, _PS, _VP, _VP, _F,
                                _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "qlora_nf4_merge": (_I32, [_I64, _I64, _I32, _PS, _VP, _VP, _F, _VP, _VP, _VP]),
    "qlora_selftest_bounded_wait": (_I32, [_I64, _VP, _VP]),
    "qlora_profile_enable": (_I32, [_I32]),
    "qlora_profile_read": (_I32, [_I32, C.POINTER(C.c_double), C.POINTER(C.c_int64)]),
    "qlora_profile_reset": (_I32, []),
    "qlora_profile_select": (_I32, [C.c_uint32]),
}

PROF_FUSED_FWD, PROF_FUSED_BWD, PROF_SKINNY, PROF_QUANTIZE = 0, 1, 2, 3
PROF_DEQUANTIZE, PROF_GEMV, PROF_OTHER = 4, 5, 6


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python bit_nf4_quantized_pack_b200/build.py` "
            "(there is no CPU or Python fallback)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if lib.qlora_abi_version() != ABI_VERSION:
        raise ImportError("libqlora_nf4.so ABI version mismatch; rebuild it")
    return lib


lib = _load()


class QLoRAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {lib.qlora_status_str(status).decode()} (status {status})"
        if status == QLORA_ERR_CUDA:
            msg += f": {lib.qlora_last_cuda_error().decode()}"
        super().__init__(msg)


def check(status: int, where: str) -> None:
    if status != QLORA_OK:
        raise QLoRAError(status, where)
