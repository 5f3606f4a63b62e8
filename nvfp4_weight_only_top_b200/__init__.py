"""NVFP4 weight-only routed-expert MoE layer for B200 (sm_100a).

Thin Python binding over the C ABI of libmoe_nvfp4.so (include/moe_nvfp4.h).  The functions
carry the C entry points' names and only marshal arguments: tensors are PyTorch CUDA tensors
(device memory and streams), every step of the layer runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _abi
from ._abi import Bank, MoeError, PackInfo, PATH_AUTO, PATH_DECODE, PATH_PREFILL  # noqa: F401
from ._abi import EP_EXPERT_MAJOR, EP_SOURCE_MAJOR  # noqa: F401

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


def _need(name: str, t, dtype, shape, device: bool = True) -> None:
    """Raises ValueError unless t is a C-contiguous tensor of this dtype and shape (and, with
    device, on the current CUDA device).  The C library takes raw pointers and the sizes of the
    bank descriptor, so a mismatch would read or write out of bounds."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and (not t.is_cuda or t.device.index != torch.cuda.current_device()):
        raise ValueError(f"{name} must be on the current CUDA device (it is on {t.device})")


def _layer_args(x, logits, bank: Bank, out, x_next=None, workspace=None, extra=()) -> int:
    """Checks the tensors of a layer call against the bank, and the (name, tensor, dtype, shape)
    entries of extra (layouts first, then devices); returns T."""
    import torch
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError("x must be a 2-D torch tensor [T, H]")
    T = int(x.shape[0])
    need = [("x", x, torch.bfloat16, (T, bank.hidden)), ("logits", logits, torch.float32, (T, bank.num_experts)),
            ("out", out, torch.bfloat16, (T, bank.hidden))]
    if x_next is not None:
        need.append(("x_next", x_next, torch.bfloat16, (T, bank.hidden)))
    if workspace is not None:
        need.append(("workspace", workspace, workspace.dtype, tuple(workspace.shape)))
    need.extend(extra(T) if callable(extra) else extra)
    for args in need:
        _need(*args, device=False)
    for args in need:
        _need(*args)
    return T


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
    if out is None and isinstance(x, torch.Tensor):
        out = torch.empty_like(x)
    T = _layer_args(x, logits, bank, out)
    _check(lib().moe_nvfp4_forward(_ptr(x), _ptr(logits), T, ctypes.byref(bank), k, _ptr(out),
                                   _stream(stream)))
    return out


def moe_nvfp4_forward_ex(x, logits, bank: Bank, k: int, out=None, x_next=None, workspace=None,
                         path: int = PATH_AUTO, stream=None):
    """As moe_nvfp4_forward, with optional residual output, caller workspace and path."""
    import torch
    if out is None and isinstance(x, torch.Tensor):
        out = torch.empty_like(x)
    T = _layer_args(x, logits, bank, out, x_next, workspace)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().moe_nvfp4_forward_ex(_ptr(x), _ptr(logits), T, ctypes.byref(bank), k, _ptr(out),
                                      _ptr(x_next), _ptr(workspace), wsb, path, _stream(stream)))
    return out


def moe_nvfp4_forward_w4a4(x, logits, bank: Bank, act_scales, k: int, out=None, x_next=None, workspace=None,
                           taps: dict | None = None, stream=None):
    """The W4A4 variant (NVFP4 activations): act_scales [E, 2] f32 device tensor holds each
    expert's input multipliers of gate/up and of down.  taps, if given, maps any of "x_codes"
    [T*k, H/2] u8, "x_scales" [T*k, H/16] u8, "h" [T*k, I] f32, "h_codes" [T*k, I/2] u8 and
    "h_scales" [T*k, I/16] u8 (device tensors) to outputs filled in slot order."""
    import torch
    if out is None and isinstance(x, torch.Tensor):
        out = torch.empty_like(x)
    H, I = bank.hidden, bank.intermediate
    for name in (taps or {}):
        if name not in ("x_codes", "x_scales", "h", "h_codes", "h_scales"):
            raise ValueError(f"unknown tap {name!r}")

    def extra(T):
        R = T * k
        shapes = {"x_codes": (torch.uint8, (R, H // 2)), "x_scales": (torch.uint8, (R, H // 16)),
                  "h": (torch.float32, (R, I)), "h_codes": (torch.uint8, (R, I // 2)),
                  "h_scales": (torch.uint8, (R, I // 16))}
        return [("act_scales", act_scales, torch.float32, (bank.num_experts, 2))] + \
               [(f"taps[{n!r}]", t, *shapes[n]) for n, t in (taps or {}).items()]

    T = _layer_args(x, logits, bank, out, x_next, workspace, extra)
    tp = _abi.W4A4Taps()
    for name, t in (taps or {}).items():
        setattr(tp, name + "_dev", t.data_ptr())
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().moe_nvfp4_forward_w4a4(_ptr(x), _ptr(logits), T, ctypes.byref(bank), _ptr(act_scales), k,
                                        _ptr(out), _ptr(x_next), _ptr(workspace), wsb, ctypes.byref(tp),
                                        _stream(stream)))
    return out


def moe_nvfp4_forward_noalloc(x, logits, bank: Bank, k: int, out=None, stream=None):
    """As moe_nvfp4_forward, with scratch from the library's fixed device array (no allocation).

    For callers that cannot allocate device memory during a call; `out` may be passed in so
    that the call itself allocates nothing on the Python side either.
    """
    import torch
    if out is None and isinstance(x, torch.Tensor):
        out = torch.empty_like(x)
    T = _layer_args(x, logits, bank, out)
    _check(lib().moe_nvfp4_forward_noalloc(_ptr(x), _ptr(logits), T, ctypes.byref(bank), k, _ptr(out),
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
    if x_host.ndim != 2 or x_host.shape[1] != bank.hidden:
        raise ValueError(f"x_host has shape {x_host.shape}, expected [T, {bank.hidden}]")
    if logits_host.shape != (x_host.shape[0], bank.num_experts):
        raise ValueError(f"logits_host has shape {logits_host.shape}, expected {(x_host.shape[0], bank.num_experts)}")
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
    if not isinstance(logits, torch.Tensor) or logits.dim() != 2:
        raise ValueError("logits must be a 2-D torch tensor [T, E]")
    T, E = (int(v) for v in logits.shape)
    _need("logits", logits, torch.float32, (T, E))
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


def moe_nvfp4_experts(x_rows, expert_ids, bank: Bank, y_rows=None, workspace=None, path: int = PATH_AUTO,
                      sorted_ids: bool = False, stream=None):
    """y_rows [R, H] f32 = expert expert_ids[r] applied to x_rows[r] (bf16 [R, H]); ids outside
    [0, E) are padding rows (zero output).  sorted_ids: the caller knows the ids are
    non-decreasing and all valid (MOE_NVFP4_EXPERTS_SORTED)."""
    import torch
    if not isinstance(x_rows, torch.Tensor) or x_rows.dim() != 2:
        raise ValueError("x_rows must be a 2-D torch tensor [R, H]")
    R = int(x_rows.shape[0])
    if y_rows is None:
        y_rows = torch.empty((R, bank.hidden), dtype=torch.float32, device=x_rows.device)
    need = [("x_rows", x_rows, torch.bfloat16, (R, bank.hidden)), ("expert_ids", expert_ids, torch.int32, (R,)),
            ("y_rows", y_rows, torch.float32, (R, bank.hidden))]
    if workspace is not None:
        need.append(("workspace", workspace, workspace.dtype, tuple(workspace.shape)))
    for args in need:
        _need(*args, device=False)
    for args in need:
        _need(*args)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().moe_nvfp4_experts(_ptr(x_rows), _ptr(expert_ids), R, ctypes.byref(bank), _ptr(y_rows),
                                   _ptr(workspace), ws_bytes, path, _abi.EXPERTS_SORTED if sorted_ids else 0,
                                   _stream(stream)))
    return y_rows


def moe_nvfp4_experts_workspace_bytes(R: int, E: int, H: int, I: int, path: int = PATH_AUTO) -> int:
    return int(lib().moe_nvfp4_experts_workspace_bytes(R, E, H, I, path))


def moe_nvfp4_gather_rows(x, perm, k: int, rows=None, stream=None):
    """rows [T*k, H] bf16 = x[perm[p] // k]: the routed rows in expert order."""
    import torch
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError("x must be a 2-D torch tensor [T, H]")
    T, H = (int(v) for v in x.shape)
    if rows is None:
        rows = torch.empty((T * k, H), dtype=torch.bfloat16, device=x.device)
    need = [("x", x, torch.bfloat16, (T, H)), ("perm", perm, torch.int32, (T * k,)),
            ("rows", rows, torch.bfloat16, (T * k, H))]
    for args in need:
        _need(*args, device=False)
    for args in need:
        _need(*args)
    _check(lib().moe_nvfp4_gather_rows(_ptr(x), _ptr(perm), T, k, H, _ptr(rows), _stream(stream)))
    return rows


def moe_nvfp4_combine(y, w, inv, k: int, out=None, x=None, x_next=None, stream=None):
    """out [T, H] bf16 = bf16(sum_j w[t, j] * y[inv[t*k+j]]), y f32 [T*k, H] in expert order."""
    import torch
    if not isinstance(w, torch.Tensor) or w.dim() != 2:
        raise ValueError("w must be a 2-D torch tensor [T, k]")
    T = int(w.shape[0])
    if not isinstance(y, torch.Tensor) or y.dim() != 2:
        raise ValueError("y must be a 2-D torch tensor [T*k, H]")
    H = int(y.shape[1])
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    need = [("y", y, torch.float32, (T * k, H)), ("w", w, torch.float32, (T, k)), ("inv", inv, torch.int32, (T * k,)),
            ("out", out, torch.bfloat16, (T, H))]
    if x_next is not None:
        need += [("x", x, torch.bfloat16, (T, H)), ("x_next", x_next, torch.bfloat16, (T, H))]
    for args in need:
        _need(*args, device=False)
    for args in need:
        _need(*args)
    _check(lib().moe_nvfp4_combine(_ptr(y), _ptr(w), _ptr(inv), T, k, H, _ptr(x if x_next is not None else None),
                                   _ptr(out), _ptr(x_next), _stream(stream)))
    return out


def moe_nvfp4_ep_plan(counts_all, rank: int, recv_rows: int, layout: int = _abi.EP_EXPERT_MAJOR, stream=None):
    """From counts_all [G, E] int32 (row s = rank s's routed rows per expert): dst_off [E] and
    recv_ids [recv_rows] (int32 CUDA tensors), as include/moe_nvfp4.h describes."""
    import torch
    if not isinstance(counts_all, torch.Tensor) or counts_all.dim() != 2:
        raise ValueError("counts_all must be a 2-D torch tensor [G, E]")
    G, E = (int(v) for v in counts_all.shape)
    _need("counts_all", counts_all, torch.int32, (G, E))
    dst_off = torch.empty(E, dtype=torch.int32, device=counts_all.device)
    recv_ids = torch.empty(max(int(recv_rows), 1), dtype=torch.int32, device=counts_all.device)
    _check(lib().moe_nvfp4_ep_plan(_ptr(counts_all), G, E, rank, layout, _ptr(dst_off), _ptr(recv_ids),
                                   int(recv_rows), _stream(stream)))
    return dst_off, recv_ids[:int(recv_rows)]


def _route_need(route: dict, T: int, k: int, E: int):
    import torch
    return [("ids", route["ids"], torch.int32, (T, k)), ("w", route["w"], torch.float32, (T, k)),
            ("perm", route["perm"], torch.int32, (T * k,)), ("inv", route["inv"], torch.int32, (T * k,)),
            ("offsets", route["offsets"], torch.int32, (E + 1,))]


def moe_nvfp4_ep_dispatch(x, route: dict, dst_off, recv_x_ptrs, capacity_rows: int, stream=None) -> None:
    """Stores this rank's routed rows (x [T, H] bf16, route = moe_nvfp4_route(...)) into their
    owners' receive buffers: recv_x_ptrs holds G device addresses (ints) valid in this process,
    each of capacity_rows rows."""
    import torch
    T, k = (int(v) for v in route["ids"].shape)
    E = int(dst_off.shape[0])
    H = int(x.shape[1])
    G = len(recv_x_ptrs)
    need = [("x", x, torch.bfloat16, (T, H)), ("dst_off", dst_off, torch.int32, (E,))] + _route_need(route, T, k, E)
    for args in need:
        _need(*args, device=False)
    for args in need:
        _need(*args)
    ptrs = (ctypes.c_void_p * G)(*[int(p) for p in recv_x_ptrs])
    _check(lib().moe_nvfp4_ep_dispatch(_ptr(x), T, k, H, E, _ptr(route["ids"]), _ptr(route["inv"]),
                                       _ptr(route["offsets"]), _ptr(dst_off), G, ptrs, int(capacity_rows),
                                       _stream(stream)))


def moe_nvfp4_ep_combine(route: dict, dst_off, recv_y_ptrs, hidden: int, capacity_rows: int, out=None, x=None,
                         x_next=None, stream=None):
    """out [T, H] bf16 = the layer's combine of the routed rows' expert outputs, read from their
    owners' f32 output buffers (recv_y_ptrs: G device addresses valid in this process, each of
    capacity_rows rows)."""
    import torch
    T, k = (int(v) for v in route["ids"].shape)
    E = int(dst_off.shape[0])
    H = int(hidden)
    G = len(recv_y_ptrs)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dst_off.device)
    need = [("dst_off", dst_off, torch.int32, (E,)), ("out", out, torch.bfloat16, (T, H))] + _route_need(route, T, k, E)
    if x_next is not None:
        need += [("x", x, torch.bfloat16, (T, H)), ("x_next", x_next, torch.bfloat16, (T, H))]
    for args in need:
        _need(*args, device=False)
    for args in need:
        _need(*args)
    ptrs = (ctypes.c_void_p * G)(*[int(p) for p in recv_y_ptrs])
    _check(lib().moe_nvfp4_ep_combine(_ptr(x if x_next is not None else None), T, k, H, E, _ptr(route["ids"]),
                                      _ptr(route["w"]), _ptr(route["inv"]), _ptr(route["offsets"]), _ptr(dst_off),
                                      G, ptrs, int(capacity_rows), _ptr(out), _ptr(x_next), _stream(stream)))
    return out


def moe_nvfp4_ep_buffer_create(nbytes: int):
    """(device address, 64-byte IPC handle) of a new peer-visible buffer on the current device."""
    p = ctypes.c_void_p()
    h = (ctypes.c_uint8 * _abi.EP_HANDLE_BYTES)()
    _check(lib().moe_nvfp4_ep_buffer_create(int(nbytes), ctypes.byref(p), h))
    return int(p.value), bytes(h)


def moe_nvfp4_ep_buffer_open(handle: bytes) -> int:
    """Device address, in this process, of another process's buffer."""
    if len(handle) != _abi.EP_HANDLE_BYTES:
        raise ValueError(f"an ep buffer handle has {_abi.EP_HANDLE_BYTES} bytes")
    p = ctypes.c_void_p()
    h = (ctypes.c_uint8 * _abi.EP_HANDLE_BYTES).from_buffer_copy(handle)
    _check(lib().moe_nvfp4_ep_buffer_open(h, ctypes.byref(p)))
    return int(p.value)


def moe_nvfp4_ep_buffer_close(peer_ptr: int) -> None:
    _check(lib().moe_nvfp4_ep_buffer_close(ctypes.c_void_p(int(peer_ptr))))


def moe_nvfp4_ep_buffer_destroy(dev_ptr: int) -> None:
    _check(lib().moe_nvfp4_ep_buffer_destroy(ctypes.c_void_p(int(dev_ptr))))


def moe_nvfp4_encode(w, dst, dst_stride: int, codes_off: int, scales_off: int, global_off: int,
                     global_mode: int = 0, stream=None) -> None:
    """NVFP4-encode n projections w [n, out, in] (bf16 CUDA tensor) into the uint8 CUDA tensor dst:
    projection i's codes, block scales and global at byte i * dst_stride + the part offsets."""
    import torch
    if not isinstance(w, torch.Tensor) or w.dim() != 3:
        raise ValueError("w must be a 3-D torch tensor [n, out, in]")
    n, out_f, in_f = (int(v) for v in w.shape)
    if not isinstance(dst, torch.Tensor) or dst.dim() != 1:
        raise ValueError("dst must be a 1-D torch uint8 tensor")
    end = max(codes_off + out_f * in_f // 2, scales_off + out_f * in_f // 16, global_off + 4)
    need = (n - 1) * dst_stride + end if n else 0
    if dst.numel() < need:
        raise ValueError(f"dst holds {dst.numel()} bytes; {need} are needed")
    for args in (("w", w, torch.bfloat16, (n, out_f, in_f)), ("dst", dst, torch.uint8, (dst.numel(),))):
        _need(*args, device=False)
    for args in (("w", w, torch.bfloat16, (n, out_f, in_f)), ("dst", dst, torch.uint8, (dst.numel(),))):
        _need(*args)
    _check(lib().moe_nvfp4_encode(_ptr(w), n, out_f, in_f, global_mode, _ptr(dst), dst_stride, codes_off,
                                  scales_off, global_off, _stream(stream)))


def record_layout(hidden: int, intermediate: int, align: int = 4096) -> dict:
    """The library's expert record: gate, up, down codes, then their block scales, then three f32
    globals, each part 16-byte aligned; records `align` bytes apart (4 KiB, as in the streaming
    pack: 22,118,412 B records every 22,122,496 B at hidden 5,120, intermediate 2,560)."""
    c = hidden * intermediate // 2
    sc = hidden * intermediate // 16
    g0 = 3 * c + 3 * sc
    rec = g0 + 12
    return {"record_bytes": rec, "record_stride": -(-rec // align) * align,
            "codes_off": (0, c, 2 * c), "scales_off": (3 * c, 3 * c + sc, 3 * c + 2 * sc),
            "global_off": (g0, g0 + 4, g0 + 8)}


def encode_bank(gate, up, down, global_mode: int = 0, stream=None):
    """A device bank from BF16 expert weights: gate and up [E, I, H], down [E, H, I] (bf16 CUDA
    tensors).  Returns (uint8 CUDA tensor holding the records, moe_nvfp4_bank)."""
    import torch
    E, I, H = (int(v) for v in gate.shape)
    if tuple(up.shape) != (E, I, H) or tuple(down.shape) != (E, H, I):
        raise ValueError("gate and up must be [E, I, H] and down [E, H, I]")
    lay = record_layout(H, I)
    buf = torch.zeros(E * lay["record_stride"], dtype=torch.uint8, device=gate.device)
    for p, w in enumerate((gate, up, down)):
        moe_nvfp4_encode(w, buf, lay["record_stride"], lay["codes_off"][p], lay["scales_off"][p],
                         lay["global_off"][p], global_mode, stream)
    bank = make_bank(buf.data_ptr(), E, H, I, lay["record_stride"], lay["codes_off"], lay["scales_off"],
                     lay["global_off"], global_mode)
    return buf, bank


def moe_nvfp4_sha256(data: bytes) -> bytes:
    """SHA-256 digest of host bytes (the digest the pack loader checks records with)."""
    buf = (ctypes.c_uint8 * 32)()
    src = ctypes.create_string_buffer(bytes(data), len(data)) if len(data) else None
    _check(lib().moe_nvfp4_sha256(src, len(data), buf))
    return bytes(buf)


class Pack:
    """An open streaming pack (moe_nvfp4_pack_open): experts.bin records and their manifest."""

    def __init__(self, manifest_path: str, bin_path: str | None = None):
        h = ctypes.c_void_p()
        _check(lib().moe_nvfp4_pack_open(manifest_path.encode(), bin_path.encode() if bin_path else None,
                                         ctypes.byref(h)))
        self.handle = h
        info = PackInfo()
        _check(lib().moe_nvfp4_pack_get_info(h, ctypes.byref(info)))
        self.info = {name: (list(getattr(info, name)) if name.endswith("_off") else getattr(info, name))
                     for name, _ in PackInfo._fields_}

    def verify(self, layer: int = -1, threads: int = 0) -> int:
        """sha256 check of the records of a layer (-1: all); returns the number that differ
        (raises MoeError with code ERR_INTEGRITY if any does)."""
        bad = ctypes.c_int64()
        rc = lib().moe_nvfp4_pack_verify(self.handle, layer, threads, ctypes.byref(bad))
        if rc == _abi.ERR_INTEGRITY:
            raise MoeError(rc, lib().moe_nvfp4_last_error().decode() + f" ({bad.value} bad)")
        _check(rc)
        return int(bad.value)

    def load(self, layer: int, dst, experts=None, dst_stride: int | None = None, verify: bool = False,
             stream=None) -> None:
        """Copies records (layer, experts[i]) (all experts if None) into the uint8 CUDA tensor dst,
        record i at byte i * dst_stride (default: the pack's record stride)."""
        import torch
        stride = int(dst_stride or self.info["record_stride"])
        n = self.info["experts"] if experts is None else len(experts)
        if n and dst.numel() < (n - 1) * stride + self.info["record_bytes"]:
            raise ValueError("dst is too small for the records")
        _need("dst", dst, torch.uint8, (dst.numel(),))
        arr = None if experts is None else (ctypes.c_int32 * n)(*[int(e) for e in experts])
        _check(lib().moe_nvfp4_pack_load(self.handle, layer, arr, n, _ptr(dst), stride, int(verify), _stream(stream)))

    def load_bank(self, layer: int, verify: bool = False, stream=None):
        """A whole layer resident on the current device: (uint8 tensor, moe_nvfp4_bank)."""
        import torch
        i = self.info
        buf = torch.empty(i["experts"] * i["record_stride"], dtype=torch.uint8, device="cuda")
        self.load(layer, buf, verify=verify, stream=stream)
        bank = make_bank(buf.data_ptr(), i["experts"], i["hidden"], i["intermediate"], i["record_stride"],
                         i["codes_off"], i["scales_off"], i["global_off"], i["global_mode"])
        return buf, bank

    def close(self) -> None:
        if self.handle:
            lib().moe_nvfp4_pack_close(self.handle)
            self.handle = None


class Rows:
    """A bounded GPU cache of one layer's expert records fed from a pack (moe_nvfp4_rows_*)."""

    def __init__(self, pack: Pack, layer: int, slots: int):
        h = ctypes.c_void_p()
        _check(lib().moe_nvfp4_rows_create(pack.handle, layer, slots, ctypes.byref(h)))
        self.handle, self.pack = h, pack

    def forward(self, x, logits, k: int, out=None, stream=None):
        import torch
        i = self.pack.info
        if out is None and isinstance(x, torch.Tensor):
            out = torch.empty_like(x)
        bank = Bank()
        bank.hidden, bank.num_experts = i["hidden"], i["experts"]
        T = _layer_args(x, logits, bank, out)
        _check(lib().moe_nvfp4_rows_forward(self.handle, _ptr(x), _ptr(logits), T, k, _ptr(out), _stream(stream)))
        return out

    def stats(self) -> dict:
        h, m, b = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib().moe_nvfp4_rows_stats(self.handle, ctypes.byref(h), ctypes.byref(m), ctypes.byref(b)))
        return {"hits": h.value, "misses": m.value, "bytes_loaded": b.value}

    def destroy(self) -> None:
        if self.handle:
            lib().moe_nvfp4_rows_destroy(self.handle)
            self.handle = None


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
