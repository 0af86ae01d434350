"""ctypes binding of librq.so (argument marshalling only).

Every step of the path runs in the library's CUDA kernels.  If the shared
library is missing this module raises at load time: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librq.so")

RQ_STATUS = {
    0: "RQ_OK",
    1: "RQ_ERR_INVALID_ARG",
    2: "RQ_ERR_UNSUPPORTED",
    3: "RQ_ERR_INFEASIBLE_BUDGET",
    4: "RQ_ERR_CAPACITY",
    5: "RQ_ERR_WORKSPACE",
    6: "RQ_ERR_CUDA",
    7: "RQ_ERR_DEVICE_TIMEOUT",
}


class RQError(RuntimeError):
    def __init__(self, func, code, msg):
        super().__init__(f"{func}: {RQ_STATUS.get(code, code)} ({msg})")
        self.code = code
        self.status = RQ_STATUS.get(code, str(code))


class CacheConfig(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int),
        ("batch", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("group", ctypes.c_int),
        ("n_sink", ctypes.c_int),
        ("n_recent", ctypes.c_int),
        ("max_tokens", ctypes.c_int),
        ("k_bits", ctypes.POINTER(ctypes.c_int)),
        ("v_bits", ctypes.POINTER(ctypes.c_int)),
        ("k_norm", ctypes.c_int),
        ("hybrid", ctypes.c_int),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_DP = ctypes.POINTER(ctypes.c_double)
_IP = ctypes.POINTER(ctypes.c_int)

# name -> (restype, argtypes); the exported C ABI of include/rq.h
SIGNATURES = {
    "rq_status_string": (ctypes.c_char_p, [_I]),
    "rq_build_info": (ctypes.c_char_p, []),
    "rq_last_cuda_error": (ctypes.c_char_p, []),
    "rq_allocate_bits": (_I, [_I, _DP, _DP, _DP, ctypes.c_double, _IP, _I, _DP, _IP, _DP]),
    "rq_measure_distortion": (_I, [_P, _I, _I, _I, _I, _IP, _I, _P, _P]),
    "rq_fit_distortion": (_I, [_I, _IP, _I, _DP, ctypes.c_double, _DP, _DP, _DP]),
    "rq_cap_weights": (_I, [_I, _DP, ctypes.c_double, _DP]),
    "rq_cache_bytes": (_I, [ctypes.POINTER(CacheConfig), ctypes.POINTER(_SZ)]),
    "rq_cache_init": (_I, [ctypes.POINTER(CacheConfig), _P, _SZ, ctypes.POINTER(_P), _P]),
    "rq_cache_destroy": (None, [_P]),
    "rq_cache_length": (_I, [_P, _I, _IP]),
    "rq_cache_stream_layout": (_I, [_P, _I, _I, _I, ctypes.POINTER(_SZ), _IP, _IP, ctypes.POINTER(_SZ)]),
    "rq_quantize_kv": (_I, [_P, _P, _P, _I, _P]),
    "rq_append_token": (_I, [_P, _I, _P, _P, _P]),
    "rq_decode_workspace_bytes": (_I, [_P, _I, ctypes.POINTER(_SZ)]),
    "rq_decode_workspace_init": (_I, [_P, _SZ, _P]),
    "rq_decode_attention": (_I, [_P, _I, _P, _P, ctypes.c_float, _I, _P, _SZ, _P]),
    "rq_decode_step": (_I, [_P, _I, _P, _P, _P, _P, ctypes.c_float, _I, _P, _SZ, _P]),
    "rq_decode_read_status": (_I, [_P, _IP]),
    "rq_selftest_device_timeout": (_I, [_P, _SZ, ctypes.c_ulonglong, _P]),
    "rq_decode_attention_noalloc": (_I, [_P, _I, _P, _P, ctypes.c_float, _I, _P]),
    "rq_decode_noalloc_read_status": (_I, [_IP]),
}

_lib = None


def lib():
    """Load librq.so once; raise if it is missing (no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} not found: build it with `python -m quantized_decode_attention_head_b200.build`"
            )
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(func: str, code: int):
    if code != 0:
        msg = lib().rq_status_string(code).decode()
        if code == 6:  # RQ_ERR_CUDA: name the CUDA error
            msg += ": " + lib().rq_last_cuda_error().decode()
        raise RQError(func, code, msg)
