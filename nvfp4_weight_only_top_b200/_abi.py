"""ctypes binding of libmoe_nvfp4.so (include/moe_nvfp4.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  Importing this module fails loudly when the
library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_nvfp4.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_WORKSPACE = -4
ERR_TIMEOUT = -5
ERR_IO = -6
ERR_INTEGRITY = -7

PATH_AUTO = 0
PATH_DECODE = 1
PATH_PREFILL = 2

EP_EXPERT_MAJOR = 0
EP_SOURCE_MAJOR = 1
EP_HANDLE_BYTES = 64
EXPERTS_SORTED = 1


class Bank(ctypes.Structure):
    """moe_nvfp4_bank."""
    _fields_ = [
        ("num_experts", ctypes.c_int32),
        ("hidden", ctypes.c_int32),
        ("intermediate", ctypes.c_int32),
        ("global_mode", ctypes.c_int32),
        ("base_dev", ctypes.c_void_p),
        ("record_stride", ctypes.c_uint64),
        ("codes_off", ctypes.c_uint64 * 3),
        ("scales_off", ctypes.c_uint64 * 3),
        ("global_off", ctypes.c_uint64 * 3),
    ]


# Every symbol include/moe_nvfp4.h declares, with its argument and return types.
_vp, _i32, _i64, _sz, _u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64
_BANKP = ctypes.POINTER(Bank)


class W4A4Taps(ctypes.Structure):
    """moe_nvfp4_w4a4_taps."""
    _fields_ = [
        ("x_codes_dev", ctypes.c_void_p),
        ("x_scales_dev", ctypes.c_void_p),
        ("h_dev", ctypes.c_void_p),
        ("h_codes_dev", ctypes.c_void_p),
        ("h_scales_dev", ctypes.c_void_p),
    ]


_TAPSP = ctypes.POINTER(W4A4Taps)
SIGNATURES = {
    "moe_nvfp4_forward": (ctypes.c_int, [_vp, _vp, _i64, _BANKP, _i32, _vp, _vp]),
    "moe_nvfp4_forward_ex": (ctypes.c_int, [_vp, _vp, _i64, _BANKP, _i32, _vp, _vp, _vp, _sz, _i32, _vp]),
    "moe_nvfp4_forward_w4a4": (ctypes.c_int, [_vp, _vp, _i64, _BANKP, _vp, _i32, _vp, _vp, _vp, _sz, _TAPSP, _vp]),
    "moe_nvfp4_forward_host": (ctypes.c_int, [_vp, _vp, _i64, _BANKP, _i32, _vp, _vp]),
    "moe_nvfp4_forward_noalloc": (ctypes.c_int, [_vp, _vp, _i64, _BANKP, _i32, _vp, _vp]),
    "moe_nvfp4_route": (ctypes.c_int, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_nvfp4_workspace_bytes": (ctypes.c_size_t, [_i64, _i32, _i32, _i32, _i32, _i32]),
    "moe_nvfp4_encode": (ctypes.c_int, [_vp, _i64, _i32, _i32, _i32, _vp, _u64, _u64, _u64, _u64, _vp]),
    "moe_nvfp4_pack_open": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_char_p, ctypes.POINTER(_vp)]),
    "moe_nvfp4_pack_get_info": (ctypes.c_int, [_vp, _vp]),
    "moe_nvfp4_pack_verify": (ctypes.c_int, [_vp, _i32, _i32, ctypes.POINTER(_i64)]),
    "moe_nvfp4_pack_load": (ctypes.c_int, [_vp, _i32, _vp, _i32, _vp, _u64, _i32, _vp]),
    "moe_nvfp4_pack_close": (ctypes.c_int, [_vp]),
    "moe_nvfp4_sha256": (ctypes.c_int, [_vp, _u64, _vp]),
    "moe_nvfp4_rows_create": (ctypes.c_int, [_vp, _i32, _i32, ctypes.POINTER(_vp)]),
    "moe_nvfp4_rows_forward": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i32, _vp, _vp]),
    "moe_nvfp4_rows_stats": (ctypes.c_int, [_vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64), ctypes.POINTER(_i64)]),
    "moe_nvfp4_rows_destroy": (ctypes.c_int, [_vp]),
    "moe_nvfp4_experts": (ctypes.c_int, [_vp, _vp, _i64, _BANKP, _vp, _vp, _sz, _i32, _i32, _vp]),
    "moe_nvfp4_experts_workspace_bytes": (ctypes.c_size_t, [_i64, _i32, _i32, _i32, _i32]),
    "moe_nvfp4_ep_plan": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _i64, _vp]),
    "moe_nvfp4_ep_dispatch": (ctypes.c_int, [_vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i64, _vp]),
    "moe_nvfp4_ep_combine": (ctypes.c_int, [_vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i64,
                                            _vp, _vp, _vp]),
    "moe_nvfp4_gather_rows": (ctypes.c_int, [_vp, _vp, _i64, _i32, _i32, _vp, _vp]),
    "moe_nvfp4_combine": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
    "moe_nvfp4_ep_buffer_create": (ctypes.c_int, [_u64, ctypes.POINTER(_vp), _vp]),
    "moe_nvfp4_ep_buffer_open": (ctypes.c_int, [_vp, ctypes.POINTER(_vp)]),
    "moe_nvfp4_ep_buffer_close": (ctypes.c_int, [_vp]),
    "moe_nvfp4_ep_buffer_destroy": (ctypes.c_int, [_vp]),
    "moe_nvfp4_last_error": (ctypes.c_char_p, []),
    "moe_nvfp4_device_status": (ctypes.c_int, []),
    "moe_nvfp4_last_launch_count": (ctypes.c_int, []),
    "moe_nvfp4_profile_begin": (ctypes.c_int, []),
    "moe_nvfp4_profile_end": (ctypes.c_int, [_vp, _vp, _i32]),
}

KERNEL_KINDS = ["route", "decode_gateup", "decode_down", "combine", "prefill_gather",
                "prefill_gateup", "prefill_down", "decode_fused", "w4a4_quant", "w4a4_gateup", "w4a4_down"]


class PackInfo(ctypes.Structure):
    """moe_nvfp4_pack_info."""
    _fields_ = [
        ("layers", ctypes.c_int32),
        ("experts", ctypes.c_int32),
        ("hidden", ctypes.c_int32),
        ("intermediate", ctypes.c_int32),
        ("record_bytes", ctypes.c_uint64),
        ("record_stride", ctypes.c_uint64),
        ("codes_off", ctypes.c_uint64 * 3),
        ("scales_off", ctypes.c_uint64 * 3),
        ("global_off", ctypes.c_uint64 * 3),
        ("global_mode", ctypes.c_int32),
        ("inexact_globals", ctypes.c_int32),
    ]


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m nvfp4_weight_only_top_b200.build` "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moe_nvfp4 error {code}: {msg}")
        self.code = code
