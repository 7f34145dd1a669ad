"""ctypes loader for ``libinfllmv2.so`` (the C ABI in include/infllmv2.h).

Argument marshalling only; every step of the computation runs in the library's CUDA
kernels.  Loading fails loudly when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libinfllmv2.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_CUDA = -4

MODE_PREFILL = 0
MODE_DECODE = 1

SCORE_SOFTMAX_SUM = 0
SCORE_LOGIT_SUM = 1
POOL_OVERLAP = 0
POOL_INSIDE = 1

OP_COMPRESS = 0
OP_SELECT_PREFILL = 1
OP_SELECT_DECODE = 2
OP_ATTN_PREFILL = 3
OP_ATTN_DECODE = 4
OP_ATTN_BACKWARD = 5

MAX_SEQ_LEN = 262144
NOALLOC_SCRATCH_BYTES = 8 << 20

# every symbol the header declares, with (restype, argtypes)
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_int = ctypes.c_int
_sz = ctypes.c_size_t


class CParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("kernel_size", ctypes.c_int32),
        ("kernel_stride", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("n_init", ctypes.c_int32),
        ("n_local", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("score_mode", ctypes.c_int32),
        ("pool_mode", ctypes.c_int32),
    ]


_P = ctypes.POINTER(CParams)
SIGNATURES = {
    "infllmv2_num_kernels": (_i64, [_P, _i64]),
    "infllmv2_compress_keys": (_int, [_P, _vp, _vp, _i32, _vp, _vp]),
    "infllmv2_select_blocks": (_int, [_P, _int, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp]),
    "infllmv2_select_blocks_chunk": (_int, [_P, _vp, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp]),
    "infllmv2_sparse_attn_prefill": (_int, [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "infllmv2_sparse_attn_chunk": (_int, [_P, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "infllmv2_sparse_attn_decode": (_int, [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "infllmv2_sparse_attn_backward": (_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz,
                                              _vp]),
    "infllmv2_sparse_attn_decode_noalloc": (_int, [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp]),
    "infllmv2_append_kv": (_int, [_P, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp]),
    "infllmv2_decode_step": (_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp]),
    "infllmv2_workspace_size": (_sz, [_P, _int, _i32]),
    "infllmv2_check_params": (_int, [_P]),
    "infllmv2_status_string": (ctypes.c_char_p, [_int]),
    "infllmv2_device_error": (_int, [_int]),
    "infllmv2_version": (_int, []),
}

_lib = None


def load(path: str = LIB_PATH):
    """Loads the library (once).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library not built: {path} is missing. Run "
                "`python -m trainable_block_sparse_compress_b200.build` (nvcc, sm_100a).")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class InfLLMv2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = load().infllmv2_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


def check(fn: str, status: int) -> None:
    if status != OK:
        raise InfLLMv2Error(fn, status)
