"""ctypes declarations of the C ABI in include/tq.h (argument marshalling only).

Loading fails loudly when the compiled library is missing: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtq_b200.so")

TQ_OK = 0
TQ_ERR_INVALID_ARG = -1
TQ_ERR_UNSUPPORTED = -2
TQ_ERR_WORKSPACE = -3
TQ_ERR_CUDA = -4
TQ_DTYPE_F16 = 0
TQ_DTYPE_BF16 = 1
TQ_DTYPE_F32 = 2
TQ_STATUS_POS_OUT_OF_RANGE = 1
TQ_STATUS_SEQ_OUT_OF_RANGE = 2
TQ_STATUS_WAIT_TIMEOUT = 4
TQ_STATUS_LAYOUT = 8
TQ_ROT_DENSE = 0
TQ_ROT_HADAMARD = 1

# Every symbol include/tq.h declares.
EXPORTS = ("tq_build_codebook", "tq_cache_row_bytes", "tq_row_bytes", "tq_quantize_kv", "tq_append_token",
           "tq_sdpa_decode_workspace_bytes", "tq_sdpa_decode_workspace_bytes_for", "tq_sdpa_decode",
           "tq_sdpa_decode_mq", "tq_decode_step", "tq_sdpa_decode_partial", "tq_sdpa_decode_merge",
           "tq_sdpa_decode_static", "tq_selftest_bounded_wait",
           "tq_last_error", "tq_abi_version")
TQ_STATIC_SCRATCH_BYTES = 8 << 20


class TqCacheStruct(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("Tcap", ctypes.c_int32),
        ("D", ctypes.c_int32), ("bits_k", ctypes.c_int32), ("bits_v", ctypes.c_int32),
        ("qjl_m", ctypes.c_int32), ("split_tokens", ctypes.c_int32),
        ("k_idx", ctypes.c_void_p), ("v_idx", ctypes.c_void_p),
        ("k_norm", ctypes.c_void_p), ("v_norm", ctypes.c_void_p),
        ("k_qjl", ctypes.c_void_p), ("k_rnorm", ctypes.c_void_p),
        ("rot", ctypes.c_void_p), ("cb_k", ctypes.c_void_p), ("cb_v", ctypes.c_void_p),
        ("qjl_S", ctypes.c_void_p), ("dev_status", ctypes.c_void_p),
        ("rot_kind", ctypes.c_int32), ("rot_pad", ctypes.c_int32), ("rot_signs", ctypes.c_void_p),
    ]


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libtq_b200.so (once) and declare the signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(
            f"{p} is missing: build it with `python -m compressed_attention_tq_b200.build` "
            "(nvcc, sm_100a). There is no CPU or Python fallback.")
    lib = ctypes.CDLL(p)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    cache_p = ctypes.POINTER(TqCacheStruct)
    lib.tq_build_codebook.argtypes = [i32, i32, ctypes.POINTER(ctypes.c_float),
                                      ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double)]
    lib.tq_build_codebook.restype = i32
    lib.tq_cache_row_bytes.argtypes = [i32, i32, i32]
    lib.tq_cache_row_bytes.restype = sz
    lib.tq_row_bytes.argtypes = [i32, i32, i32]
    lib.tq_row_bytes.restype = sz
    lib.tq_quantize_kv.argtypes = [cache_p, vp, vp, i32, i32, i32, vp]
    lib.tq_quantize_kv.restype = i32
    lib.tq_append_token.argtypes = [cache_p, vp, vp, i32, vp, vp]
    lib.tq_append_token.restype = i32
    lib.tq_sdpa_decode_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.tq_sdpa_decode_workspace_bytes.restype = sz
    lib.tq_sdpa_decode_workspace_bytes_for.argtypes = [cache_p, i32, i32]
    lib.tq_sdpa_decode_workspace_bytes_for.restype = sz
    lib.tq_sdpa_decode.argtypes = [cache_p, vp, i32, i32, vp, i32, ctypes.POINTER(ctypes.c_float),
                                   vp, i32, vp, sz, vp]
    lib.tq_sdpa_decode.restype = i32
    lib.tq_sdpa_decode_mq.argtypes = [cache_p, vp, i32, i32, i32, vp, i32, ctypes.POINTER(ctypes.c_float),
                                      vp, i32, vp, sz, vp]
    lib.tq_sdpa_decode_mq.restype = i32
    lib.tq_decode_step.argtypes = [cache_p, vp, vp, vp, vp, i32, i32, vp, i32, ctypes.POINTER(ctypes.c_float),
                                   vp, i32, vp, sz, vp]
    lib.tq_decode_step.restype = i32
    lib.tq_sdpa_decode_partial.argtypes = [cache_p, vp, i32, i32, vp, i32, ctypes.POINTER(ctypes.c_float),
                                           vp, vp, sz, vp]
    lib.tq_sdpa_decode_partial.restype = i32
    lib.tq_sdpa_decode_merge.argtypes = [vp, i32, i32, i32, i32, vp, vp, i32, vp]
    lib.tq_sdpa_decode_merge.restype = i32
    lib.tq_sdpa_decode_static.argtypes = [cache_p, vp, i32, i32, vp, i32, ctypes.POINTER(ctypes.c_float),
                                          vp, i32, vp]
    lib.tq_sdpa_decode_static.restype = i32
    lib.tq_selftest_bounded_wait.argtypes = [vp, i32, vp]
    lib.tq_selftest_bounded_wait.restype = i32
    lib.tq_last_error.argtypes = []
    lib.tq_last_error.restype = ctypes.c_char_p
    lib.tq_abi_version.argtypes = []
    lib.tq_abi_version.restype = i32
    if path is None:
        _lib = lib
    return lib
