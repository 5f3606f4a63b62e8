"""Device-side writer of synthetic banks (libmoe_inputs.so, built from fill.cu).

Writes the same bytes as gen.record_bytes() for every record, for banks too large to build
on the host (a 24-layer stack is ~136 GB).
"""
from __future__ import annotations

import ctypes
import os

from .gen import RecordLayout, global_value

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_inputs.so")
_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} missing: run `python -m nvfp4_weight_only_top_b200.build`")
        _LIB = ctypes.CDLL(_LIB_PATH)
        _LIB.moe_inputs_fill_bank.restype = ctypes.c_int
        _LIB.moe_inputs_fill_bank.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_float, ctypes.c_void_p]
        _LIB.moe_inputs_stream_key.restype = ctypes.c_uint64
        _LIB.moe_inputs_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
    return _LIB


def stream_key_native(seed: int, layer: int, expert: int, stream: int) -> int:
    return int(lib().moe_inputs_stream_key(seed, layer, expert, stream))


def fill_bank(base_ptr: int, lay: RecordLayout, seed: int, layer: int, global_mode: int = 0,
              stream_ptr: int = 0) -> None:
    """Writes all lay.E records of (seed, layer) at device address base_ptr."""
    assert lay.codes_off == (0, lay.I * lay.H // 2, lay.I * lay.H)       # the layout fill.cu writes
    rc = lib().moe_inputs_fill_bank(ctypes.c_void_p(base_ptr), lay.record_stride, lay.H, lay.I, seed, layer, 0,
                                    lay.E, float(global_value(lay.H, global_mode)), ctypes.c_void_p(stream_ptr))
    if rc != 0:
        raise RuntimeError(f"moe_inputs_fill_bank failed with CUDA error {rc}")


def bank_tensor(lay: RecordLayout, seed: int, layer: int, global_mode: int = 0, device: str = "cuda"):
    """A torch uint8 CUDA tensor holding the whole bank of (seed, layer)."""
    import torch
    buf = torch.empty(lay.bank_bytes, dtype=torch.uint8, device=device)
    fill_bank(buf.data_ptr(), lay, seed, layer, global_mode, torch.cuda.current_stream().cuda_stream)
    return buf
