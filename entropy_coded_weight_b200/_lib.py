"""ctypes binding of libeqw.so (include/eqw.h): argument marshalling only.

Every entry point keeps its C name.  The library is loaded from this package's
directory (or from the path in EQW_LIBRARY); if it is missing the import fails loudly (there is no CPU
fallback: decoding only runs in the CUDA kernels of libeqw).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# EQW_LIBRARY selects another build of the same library, e.g. libeqw_checked.so
LIB_PATH = os.environ.get("EQW_LIBRARY") or os.path.join(HERE, "libeqw.so")

EQ_OK, EQ_ERR_INVALID_ARG, EQ_ERR_CORRUPT, EQ_ERR_UNSUPPORTED = 0, 1, 2, 3
EQ_ERR_CUDA, EQ_ERR_TIMEOUT, EQ_ERR_NOSPACE = 4, 5, 6
EQ_DEV_BAD_HEADER, EQ_DEV_BAD_TABLE, EQ_DEV_BAD_STATE = 1, 2, 4
EQ_DEV_BAD_END, EQ_DEV_TIMEOUT, EQ_DEV_BAD_OUTLIER, EQ_DEV_CHECK = 8, 16, 32, 64
EQ_INT8, EQ_E4M3 = 1, 2
EQ_TABLE_PER_CHUNK = 1
EQ_CODEC_HUFFMAN = 2


class EqError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = _lib.eq_status_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{what}: {msg} (status {code})")


class eq_matrix_in(ctypes.Structure):
    _fields_ = [
        ("layer", ctypes.c_uint32),
        ("dtype", ctypes.c_uint32),
        ("rows", ctypes.c_uint32),
        ("cols", ctypes.c_uint32),
        ("symbols", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("n_out", ctypes.c_uint32),
        ("out_row", ctypes.c_void_p),
        ("out_col", ctypes.c_void_p),
        ("out_val", ctypes.c_void_p),
        ("flags", ctypes.c_uint32),
    ]


class eq_matrix_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint32) for n in
                ("layer", "index", "dtype", "rows", "cols", "n_chunks", "n_outliers", "uniform_table",
                 "codec", "reserved")] + [
        ("compressed_bytes", ctypes.c_uint64),
        ("payload_words", ctypes.c_uint64),
    ]


# name -> (restype, argtypes)
_vp, _u32, _u64, _i32, _sz = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int, ctypes.c_size_t
_P = ctypes.POINTER
SIGNATURES = {
    "eq_encoder_run": (_i32, [_P(eq_matrix_in), _u32, _i32, _P(_vp), _P(_sz)]),
    "eq_encoded_write": (_i32, [_vp, _vp, _sz]),
    "eq_encoded_free": (None, [_vp]),
    "eq_encode_host": (_i32, [_P(eq_matrix_in), _u32, _i32, _vp, _sz, _P(_sz)]),
    "eq_model_open": (_i32, [_vp, _sz, _vp, _P(_vp)]),
    "eq_model_close": (None, [_vp]),
    "eq_model_set_sm_limit": (_i32, [_vp, ctypes.c_uint32]),
    "eq_model_counts": (_i32, [_vp, _P(_u32), _P(_u32)]),
    "eq_matrix_get_info": (_i32, [_vp, _u32, _P(eq_matrix_info)]),
    "eq_layer_matrices": (_i32, [_vp, _u32, _P(_u32), _P(_u32)]),
    "eq_block_layout": (_i32, [_vp, _u32, _P(_sz), _u32, _P(_sz)]),
    "eq_decode_plan": (_i32, [_vp, _u32, _u32, _P(_u32), _u32]),
    "eq_decode_matrix": (_i32, [_vp, _u32, _vp, _sz, _vp, _vp]),
    "eq_decode_block": (_i32, [_vp, _u32, _vp, _sz, _vp, _vp]),
    "eq_decode_model_stream": (_i32, [_vp, _u32, _P(_vp), _sz, _vp, _vp, _P(_vp), _P(_vp)]),
    "eq_gemv_bf16": (_i32, [_vp, _vp, _vp, _u32, _u32, _vp]),
    "eq_encode_device": (_i32, [_vp, _u32, _vp, _sz, _vp, _vp, _sz, _vp]),
    "eq_encode_device_workspace": (_i32, [_vp, _u32, _vp]),
    "eq_encode_device_noalloc": (_i32, [_vp, _u32, _vp, _sz, _vp, _vp]),
    "eq_encode_bound": (_i32, [_vp, _u32, _vp]),
    "eq_decode_gemv_matrix": (_i32, [_vp, _u32, _vp, _vp, _vp, _vp]),
    "eq_decode_gemv_block": (_i32, [_vp, _u32, _vp, _vp, _u32, _vp, _vp]),
    "eq_decode_symbols": (_i32, [_vp, _u32, _vp, _sz, _vp, _vp]),
    "eq_decode_symbols_block": (_i32, [_vp, _u32, _vp, _u32, _vp, _vp]),
    "eq_gemm_symbols": (_i32, [_vp, _u32, _vp, _vp, _u32, _vp, _vp, _vp]),
    "eq_gemm_symbols_block": (_i32, [_vp, _u32, _vp, _vp, _u32, _vp, _u32, _vp, _vp]),
    "eq_selftest_wait_timeout": (_i32, [_vp, _vp]),
    "eq_selftest_gemm_wait_timeout": (_i32, [_vp, _vp]),
    "eq_status_string": (ctypes.c_char_p, [_i32]),
    "eq_format_version": (_i32, []),
    "eq_build_checked": (_i32, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libeqw.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libeqw.so not built ({LIB_PATH}); run "
                              "`python -m entropy_coded_weight_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(code: int, what: str) -> None:
    if code != EQ_OK:
        raise EqError(code, what)
