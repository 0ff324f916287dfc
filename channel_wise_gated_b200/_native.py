"""ctypes binding of the C ABI in include/kda.h (libkda_b200.so, built in-tree).

This module only loads the library and declares the entry points' signatures.
There is no fallback: if the library is missing or fails to load, every call
raises.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda_b200.so")

KDA_F32 = 0
KDA_BF16 = 1

KDA_OK = 0
KDA_ERR_NULL = -1
KDA_ERR_SHAPE = -2
KDA_ERR_DTYPE = -3
KDA_ERR_ALIGN = -4
KDA_ERR_SEQLENS = -5
KDA_ERR_CUDA = -6
KDA_ERR_TIMEOUT = -7
KDA_ERR_SCRATCH = -8

KDA_DECODE_MAX_TOKENS = 16
KDA_MAX_SEGMENTS = 64
SIZE_MAX = ctypes.c_size_t(-1).value

# entry point -> argument types (all return int except kda_status_string)
_P, _I32, _I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
SIGNATURES = {
    "kda_chunk_fwd": [_P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P, _P],
    "kda_chunk_fwd_simt": [_P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P, _P],
    "kda_chunk_fwd_ws": [_P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P, _P,
                         ctypes.c_size_t, _P],
    "kda_chunk_fwd_workspace_size": [_I32, _I64, _I32, ctypes.c_int, ctypes.c_int],
    "kda_chunk_fwd_split_plan": [_I32, _I64, _I32, ctypes.c_size_t, _P],
    "kda_chunk_fwd_static": [_P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P, _P],
    "kda_chunk_fwd_fused": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, _P, _P, _P,
                            ctypes.c_size_t, _P],
    "kda_dplr_chunk_fwd": [_P, _P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P,
                           _P],
    "kda_short_conv_swish": [_P, _P, _P, _I32, _I64, _I32, _P, _P],
    "kda_gdn_chunk_fwd": [_P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P, _P],
    "kda_gdn_chunk_fwd_ws": [_P, _P, _P, _P, _P, _P, _P, _I32, _I64, _I32, ctypes.c_int, _P, _P, _P,
                             ctypes.c_size_t, _P],
    "kda_decode_step": [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, ctypes.c_int, ctypes.c_int, _P],
    "kda_decode_tokens": [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, ctypes.c_int, ctypes.c_int,
                          _P],
    "kda_testing_chunk_fwd_stall": [_P, _P, _P, _P, _P, _P, _I64, _I32, _P, _P, _I32, ctypes.c_uint32,
                                    _P],
    "kda_device_status": [_P],
    "kda_status_string": [ctypes.c_int],
}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load(path: str = LIB_PATH):
    """Load the library (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"KDA CUDA library not found at {path}; build it with "
            "`python -m channel_wise_gated_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, argtypes in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = {"kda_status_string": ctypes.c_char_p,
                      "kda_chunk_fwd_workspace_size": ctypes.c_size_t}.get(name, ctypes.c_int)
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != KDA_OK:
        raise KdaError(status, where)
