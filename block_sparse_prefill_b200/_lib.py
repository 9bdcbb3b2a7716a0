"""ctypes declarations of the C ABI in include/fp2.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp2.so")

FP2_BF16 = 0
FP2_E4M3 = 1

STATUS = {
    0: "FP2_OK", 1: "FP2_ERR_INVALID_ARG", 2: "FP2_ERR_UNSUPPORTED", 3: "FP2_ERR_WORKSPACE",
    4: "FP2_ERR_CUDA", 5: "FP2_ERR_TIMEOUT", 6: "FP2_ERR_BAD_INDEX",
}

# every function the header declares
EXPORTS = ["fp2_max_blocks", "fp2_workspace_bytes", "fp2_workspace_init", "fp2_estimate",
           "fp2_sparse_prefill", "fp2_prefill_paged", "fp2_get_error", "fp2_status_string",
           "fp2_version", "fp2_sparse_prefill_noalloc", "fp2_estimate_chunked", "fp2_prefill_chunked"]

NOALLOC_SCRATCH_BYTES = 8 << 20  # FP2_NOALLOC_SCRATCH_BYTES


class fp2_params(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("alpha", ctypes.c_float),
        ("sm_scale", ctypes.c_float),
        ("correction", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("q_scale", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
    ]


class fp2_blockmeta(ctypes.Structure):
    _fields_ = [
        ("kept_cnt", ctypes.c_void_p),
        ("kept_idx", ctypes.c_void_p),
        ("k_mean", ctypes.c_void_p),
        ("v_mean", ctypes.c_void_p),
        ("score_dbg", ctypes.c_void_p),
        ("nb_max", ctypes.c_int32),
        ("max_blocks", ctypes.c_int32),
        ("k_var", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_PP = ctypes.POINTER(fp2_params)
_PM = ctypes.POINTER(fp2_blockmeta)

_lib = None


def load():
    """Loads libfp2.so; raises when it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m block_sparse_prefill_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.fp2_max_blocks.argtypes = [_I32, _I64, _I32]
    lib.fp2_max_blocks.restype = _I64
    lib.fp2_workspace_bytes.argtypes = [_PP, _I32, _I64, _I32]
    lib.fp2_workspace_bytes.restype = _SZ
    lib.fp2_workspace_init.argtypes = [_P, _SZ, _P]
    lib.fp2_workspace_init.restype = ctypes.c_int
    lib.fp2_estimate.argtypes = [_PP, _P, _P, _P, _P, _I32, _I64, _I32, _P, _I32, _I32, _PM, _P, _SZ, _P]
    lib.fp2_estimate.restype = ctypes.c_int
    lib.fp2_sparse_prefill.argtypes = [_PP, _P, _P, _P, _P, _I32, _I64, _I32, _PM, _P, _P, _P, _SZ, _P]
    lib.fp2_sparse_prefill.restype = ctypes.c_int
    lib.fp2_prefill_paged.argtypes = [_PP, _P, _P, _P, _P, _I32, _I64, _I32, _P, _I32, _I32, _PM, _P, _P,
                                      _P, _SZ, _P]
    lib.fp2_prefill_paged.restype = ctypes.c_int
    lib.fp2_estimate_chunked.argtypes = [_PP, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I32, _P, _I32, _I32, _PM,
                                         _P, _SZ, _P]
    lib.fp2_estimate_chunked.restype = ctypes.c_int
    lib.fp2_prefill_chunked.argtypes = [_PP, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I32, _P, _I32, _I32, _PM,
                                        _P, _P, _P, _SZ, _P]
    lib.fp2_prefill_chunked.restype = ctypes.c_int
    lib.fp2_get_error.argtypes = [_P, _P]
    lib.fp2_get_error.restype = ctypes.c_int
    lib.fp2_status_string.argtypes = [ctypes.c_int]
    lib.fp2_status_string.restype = ctypes.c_char_p
    lib.fp2_sparse_prefill_noalloc.argtypes = [_PP, _P, _P, _P, _P, _I32, _I64, _I32, _PM, _P, _P, _P, _P]
    lib.fp2_sparse_prefill_noalloc.restype = ctypes.c_int
    lib.fp2_version.argtypes = []
    lib.fp2_version.restype = _I32
    _lib = lib
    return lib
