"""NVFP4 weight-only routed-expert MoE layer for B200 (sm_100a).

Thin Python binding over the C ABI of libmoe_nvfp4.so (include/moe_nvfp4.h).  The functions
carry the C entry points' names and only marshal arguments: tensors are PyTorch CUDA tensors
(device memory and streams), every step of the layer runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _abi
from ._abi import Bank, MoeError, PATH_AUTO, PATH_DECODE, PATH_PREFILL  # noqa: F401

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises ImportError if it has not been built)."""
    global _LIB
    if _LIB is None:
        _LIB = _abi.load()
    return _LIB


def _check(rc: int) -> None:
    if rc != _abi.OK:
        raise MoeError(rc, lib().moe_nvfp4_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream.cuda_stream)


def make_bank(base_ptr: int, num_experts: int, hidden: int, intermediate: int, record_stride: int,
              codes_off, scales_off, global_off, global_mode: int = 0) -> Bank:
    """moe_nvfp4_bank for E records at device address base_ptr."""
    b = Bank()
    b.num_experts, b.hidden, b.intermediate, b.global_mode = num_experts, hidden, intermediate, global_mode
    b.base_dev = ctypes.c_void_p(int(base_ptr))
    b.record_stride = record_stride
    for p in range(3):
        b.codes_off[p], b.scales_off[p], b.global_off[p] = codes_off[p], scales_off[p], global_off[p]
    return b


def moe_nvfp4_forward(x, logits, bank: Bank, k: int, out=None, stream=None):
    """out [T, H] bf16 = MoE(x [T, H] bf16, logits [T, E] f32) on the current device."""
    import torch
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    _check(lib().moe_nvfp4_forward(_ptr(x), _ptr(logits), T, ctypes.byref(bank), k, _ptr(out),
                                   _stream(stream)))
    return out


def moe_nvfp4_forward_ex(x, logits, bank: Bank, k: int, out=None, x_next=None, workspace=None,
                         path: int = PATH_AUTO, stream=None):
    """As moe_nvfp4_forward, with optional residual output, caller workspace and path."""
    import torch
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().moe_nvfp4_forward_ex(_ptr(x), _ptr(logits), T, ctypes.byref(bank), k, _ptr(out),
                                      _ptr(x_next), _ptr(workspace), wsb, path, _stream(stream)))
    return out


def moe_nvfp4_forward_noalloc(x, logits, bank: Bank, k: int, out=None, stream=None):
    """As moe_nvfp4_forward, with scratch from the library's fixed device array (no allocation).

    For callers that cannot allocate device memory during a call; `out` may be passed in so
    that the call itself allocates nothing on the Python side either.
    """
    import torch
    if out is None:
        out = torch.empty_like(x)
    _check(lib().moe_nvfp4_forward_noalloc(_ptr(x), _ptr(logits), x.shape[0], ctypes.byref(bank), k, _ptr(out),
                                           _stream(stream)))
    return out


def moe_nvfp4_forward_host(x_host: np.ndarray, logits_host: np.ndarray, bank: Bank, k: int,
                           out_host: np.ndarray | None = None, stream=None) -> np.ndarray:
    """End-to-end call on host arrays: x [T, H] BF16 bit patterns (uint16), logits [T, E] f32.

    Returns out [T, H] as BF16 bit patterns (uint16).  Host arrays may be pinned (e.g. numpy
    views of pinned torch tensors) for asynchronous copies.
    """
    x_host = np.ascontiguousarray(x_host, dtype=np.uint16)
    logits_host = np.ascontiguousarray(logits_host, dtype=np.float32)
    if out_host is None:
        out_host = np.empty_like(x_host)
    elif out_host.dtype != np.uint16 or not out_host.flags.c_contiguous or out_host.shape != x_host.shape:
        raise ValueError("out_host must be a C-contiguous uint16 array shaped like x_host")
    # (ctypes.c_void_p of the integer address: a third of the cost of ndarray.ctypes.data_as)
    _check(lib().moe_nvfp4_forward_host(ctypes.c_void_p(x_host.ctypes.data), ctypes.c_void_p(logits_host.ctypes.data),
                                        x_host.shape[0], ctypes.byref(bank), k,
                                        ctypes.c_void_p(out_host.ctypes.data), _stream(stream)))
    return out_host


def moe_nvfp4_route(logits, k: int, stream=None) -> dict:
    """Routing only: ids, w, counts, offsets, perm, inv (int32 / f32 CUDA tensors)."""
    import torch
    T, E = logits.shape
    dev = logits.device
    r = dict(ids=torch.empty((T, k), dtype=torch.int32, device=dev),
             w=torch.empty((T, k), dtype=torch.float32, device=dev),
             counts=torch.empty(E, dtype=torch.int32, device=dev),
             offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
             perm=torch.empty(T * k, dtype=torch.int32, device=dev),
             inv=torch.empty(T * k, dtype=torch.int32, device=dev))
    _check(lib().moe_nvfp4_route(_ptr(logits), T, E, k, _ptr(r["ids"]), _ptr(r["w"]), _ptr(r["counts"]),
                                 _ptr(r["offsets"]), _ptr(r["perm"]), _ptr(r["inv"]), _stream(stream)))
    return r


def moe_nvfp4_workspace_bytes(T: int, E: int, k: int, H: int, I: int, path: int = PATH_AUTO) -> int:
    return int(lib().moe_nvfp4_workspace_bytes(T, E, k, H, I, path))


def moe_nvfp4_device_status() -> int:
    return int(lib().moe_nvfp4_device_status())


def moe_nvfp4_last_launch_count() -> int:
    return int(lib().moe_nvfp4_last_launch_count())


def moe_nvfp4_last_error() -> str:
    return lib().moe_nvfp4_last_error().decode()


def moe_nvfp4_profile_begin() -> None:
    _check(lib().moe_nvfp4_profile_begin())


def moe_nvfp4_profile_end() -> dict:
    """{kernel kind: (summed ms, launches)} of the bracketed launches (see the header)."""
    n = len(_abi.KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(lib().moe_nvfp4_profile_end(ms, cnt, n))
    return {name: (ms[i], cnt[i]) for i, name in enumerate(_abi.KERNEL_KINDS) if cnt[i]}
