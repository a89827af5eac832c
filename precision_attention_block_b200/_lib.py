"""ctypes view of libthrift's C ABI (include/thrift.h, include/thrift_debug.h).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.  If the
library is missing or cannot be loaded, loading raises -- there is no other code path.
"""

from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
# THRIFT_LIB selects another build of the same ABI (e.g. libthrift_checked.so, the checked build)
LIB_PATH = os.environ.get("THRIFT_LIB") or os.path.join(HERE, "libthrift.so")

THRIFT_OK = 0
THRIFT_ERR_INVALID_ARG = 1
THRIFT_ERR_UNSUPPORTED = 2
THRIFT_ERR_CUDA = 3
THRIFT_ERR_TIMEOUT = 4
THRIFT_ERR_WORKSPACE = 5
THRIFT_ERR_CHECK = 8


class ThriftError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


class CCfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
                ("topk_abs", ctypes.c_int32), ("topk_bp", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class CDecodeCfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("Nq", ctypes.c_int32), ("Nk", ctypes.c_int32), ("d", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("block_k", ctypes.c_int32),
                ("topk_abs", ctypes.c_int32), ("topk_bp", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("n_valid", ctypes.c_int32)]


class CStrides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("n", ctypes.c_int64)]


class CNVFP4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("scales_mma", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("group_axis", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_cfgp = ctypes.POINTER(CCfg)
_nvp = ctypes.POINTER(CNVFP4)
_dcfgp = ctypes.POINTER(CDecodeCfg)
_stp = ctypes.POINTER(CStrides)

SIGNATURES = {
    "thrift_nvfp4_scales_mma_bytes": (_sz, [_i64, _i32, _i32, _i32]),
    "thrift_workspace_bytes": (_sz, [_cfgp]),
    "thrift_auto_workspace_bytes": (_sz, [_cfgp]),
    "thrift_quantize_nvfp4": (ctypes.c_int, [_vp, _i64, _i32, _i32, _nvp, _vp, _sz, _vp]),
    "thrift_block_select": (ctypes.c_int, [_vp, _vp, _cfgp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "thrift_block_select_noalloc": (ctypes.c_int, [_vp, _vp, _cfgp, _vp, _vp, _vp, _vp, _vp]),
    "thrift_attn_fwd": (ctypes.c_int, [_vp, _vp, _vp, _nvp, _nvp, _nvp, _vp, _vp, _vp, _vp, _vp, _cfgp,
                                       _vp, _sz, _vp]),
    "thrift_attn_fwd_auto": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _cfgp, _vp, _sz, _vp]),
    "thrift_attn_fwd_qat": (ctypes.c_int, [_vp, _vp, _vp, _nvp, _nvp, _nvp, _vp, _vp, _vp, _vp, _cfgp, _vp, _sz,
                                           _vp]),
    "thrift_attn_fwd_running_max": (ctypes.c_int, [_vp, _vp, _vp, _nvp, _nvp, _nvp, _vp, _vp, _vp, _cfgp, _vp,
                                                   _sz, _vp]),
    "thrift_quantize_nvfp4_strided": (ctypes.c_int, [_vp, _stp, _i32, _i32, _i32, _i32, _nvp, _vp, _sz, _vp]),
    "thrift_block_select_strided": (ctypes.c_int, [_vp, _stp, _vp, _stp, _cfgp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "thrift_attn_fwd_strided": (ctypes.c_int, [_vp, _stp, _vp, _stp, _vp, _stp, _nvp, _nvp, _nvp, _vp, _vp, _stp,
                                               _vp, _cfgp, _vp, _sz, _vp]),
    "thrift_attn_fwd_auto_strided": (ctypes.c_int, [_vp, _stp, _vp, _stp, _vp, _stp, _vp, _stp, _vp, _cfgp, _vp,
                                                    _sz, _vp]),
    "thrift_kv_block_means": (ctypes.c_int, [_vp, _i64, _i32, _i32, _i32, _vp, _vp]),
    "thrift_nvfp4_tensor_scale": (ctypes.c_int, [_vp, _i64, _vp, _vp, _sz, _vp]),
    "thrift_kv_append": (ctypes.c_int, [_vp, _vp, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _nvp, _nvp, _vp,
                                        _vp]),
    "thrift_decode_workspace_bytes": (_sz, [_dcfgp]),
    "thrift_decode_select": (ctypes.c_int, [_vp, _vp, _dcfgp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "thrift_decode_attn": (ctypes.c_int, [_vp, _vp, _vp, _nvp, _nvp, _vp, _vp, _vp, _dcfgp, _vp, _sz, _vp]),
    "thrift_decode_attn_sparse": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _dcfgp, _vp, _sz, _vp]),
    "thrift_attn_fwd_sparse": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _cfgp, _vp, _sz, _vp]),
    "thrift_decode_fwd": (ctypes.c_int, [_vp, _vp, _vp, _nvp, _nvp, _vp, _vp, _vp, _dcfgp, _vp, _sz, _vp]),
    "thrift_reset_device_status": (ctypes.c_int, [_vp, _vp]),
    "thrift_get_device_status": (ctypes.c_int, [_vp, _vp, ctypes.POINTER(_i32)]),
    "thrift_debug_wait_timeout": (ctypes.c_int, [_vp, _i64, _vp]),
    "thrift_debug_ex2": (ctypes.c_int, [_vp, _vp, _i64, _i32, _vp]),
    "thrift_debug_pipe_rates_ws_bytes": (_sz, []),
    "thrift_debug_pipe_rates": (ctypes.c_int, [_vp, _sz, _vp, _vp]),
    "thrift_debug_checks_enabled": (ctypes.c_int32, []),
    "thrift_debug_check": (ctypes.c_int, [_vp, _i32, _vp]),
    "thrift_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "thrift_debug_attn_dump": (ctypes.c_int, [_vp, _vp, _vp, _nvp, _nvp, _nvp, _vp, _vp, _vp, _cfgp, _vp,
                                              _sz, _vp, _i32, _vp]),
}


def load():
    """The loaded library.  Raises if libthrift.so has not been built (run build())."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build the CUDA library first "
                    "(python -m precision_attention_block_b200.build)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_str(status: int) -> str:
    try:
        return load().thrift_status_str(status).decode()
    except ImportError:
        return "unknown"


def check(status: int, what: str) -> None:
    if status != THRIFT_OK:
        raise ThriftError(status, what)
