"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export every entry point the header declares, and reject invalid
arguments on the host before touching a device.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import moe_inputs
from moe_inputs import device as mdev
import nvfp4_weight_only_top_b200 as moe
from nvfp4_weight_only_top_b200 import _abi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe_nvfp4.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_nvfp4_\w+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = _declared()
    assert "moe_nvfp4_forward" in names and "moe_nvfp4_route" in names
    assert set(names) == set(_abi.SIGNATURES), "binding signatures must cover the header exactly"


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_abi.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    moe.lib()       # typed load succeeds


def test_bank_struct_layout_matches_header():
    assert ctypes.sizeof(_abi.Bank) == 4 * 4 + 8 + 8 + 3 * 8 * 3
    assert _abi.Bank.base_dev.offset == 16 and _abi.Bank.codes_off.offset == 32


def _bank(**kw):
    lay = moe_inputs.record_layout(16, 256, 128)
    args = dict(base_ptr=0x10000, num_experts=16, hidden=256, intermediate=128,
                record_stride=lay.record_stride, codes_off=lay.codes_off, scales_off=lay.scales_off,
                global_off=lay.global_off, global_mode=0)
    args.update(kw)
    return moe.make_bank(**args)


def _fwd(bank, T=4, k=2, x=0x20000, lg=0x30000, out=0x40000):
    lib = moe.lib()
    return lib.moe_nvfp4_forward(ctypes.c_void_p(x), ctypes.c_void_p(lg), T,
                                 ctypes.byref(bank) if bank is not None else None, k, ctypes.c_void_p(out), None)


@pytest.mark.parametrize("kw,code", [
    (dict(num_experts=0), _abi.ERR_UNSUPPORTED),
    (dict(num_experts=2048), _abi.ERR_UNSUPPORTED),
    (dict(hidden=200), _abi.ERR_UNSUPPORTED),
    (dict(intermediate=64), _abi.ERR_UNSUPPORTED),
    (dict(global_mode=2), _abi.ERR_INVALID_ARG),
    (dict(base_ptr=0x10008), _abi.ERR_INVALID_ARG),
    (dict(record_stride=1000), _abi.ERR_INVALID_ARG),
])
def test_bank_validation(kw, code):
    assert _fwd(_bank(**kw)) == code
    assert moe.moe_nvfp4_last_error() != ""


def test_null_bank_and_bad_k_and_T():
    assert _fwd(None) == _abi.ERR_INVALID_ARG
    assert _fwd(_bank(), k=0) == _abi.ERR_INVALID_ARG
    assert _fwd(_bank(), k=17) == _abi.ERR_INVALID_ARG        # k > E
    assert _fwd(_bank(), k=33) == _abi.ERR_INVALID_ARG
    assert _fwd(_bank(), T=-1) == _abi.ERR_INVALID_ARG
    assert "T = -1" in moe.moe_nvfp4_last_error()


def test_workspace_bytes_is_host_only():
    a = moe.moe_nvfp4_workspace_bytes(1, 256, 8, 5120, 2560)
    b = moe.moe_nvfp4_workspace_bytes(64, 256, 8, 5120, 2560)
    assert 0 < a < b
    assert moe.moe_nvfp4_workspace_bytes(-1, 256, 8, 5120, 2560) == 0
    assert moe.moe_nvfp4_workspace_bytes(1, 256, 0, 5120, 2560) == 0
    # the h and y buffers dominate: R*(H+I)*4
    assert b >= 64 * 8 * (5120 + 2560) * 4


def test_input_generator_key_matches_native():
    for args in [(0, 0, 0, 0), (7, 3, 255, 1), (123456789, 23, 17, 0)]:
        assert mdev.stream_key_native(*args) == moe_inputs.gen.stream_key(*args)


def _fwd_ex(bank, T=4, k=2, path=_abi.PATH_AUTO):
    lib = moe.lib()
    return lib.moe_nvfp4_forward_ex(ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), T, ctypes.byref(bank), k,
                                    ctypes.c_void_p(0x40000), None, None, 0, path, None)


def test_unknown_path_and_oversized_T_are_rejected_on_the_host():
    assert _fwd_ex(_bank(), path=3) == _abi.ERR_INVALID_ARG
    assert _fwd_ex(_bank(), path=-1) == _abi.ERR_INVALID_ARG
    assert "path" in moe.moe_nvfp4_last_error()
    assert _fwd_ex(_bank(), T=1 << 40) == _abi.ERR_UNSUPPORTED


@pytest.mark.parametrize("part", [0, 1, 2])
def test_projection_offsets_are_validated(part):
    lay = moe_inputs.record_layout(16, 256, 128)
    for field, bad in (("codes_off", 8), ("scales_off", 4), ("global_off", 2)):
        offs = list(getattr(lay, field))
        offs[part] += bad
        assert _fwd(_bank(**{field: offs})) == _abi.ERR_INVALID_ARG, (field, part)
    offs = list(lay.codes_off)
    offs[part] = lay.record_stride                    # starts past the end of the record
    assert _fwd(_bank(codes_off=offs)) == _abi.ERR_INVALID_ARG


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the behaviour without a CUDA device")
def test_valid_call_without_a_device_fails_loudly():
    """No CPU fallback: with every argument valid and no CUDA device, the call returns an error."""
    assert _fwd(_bank()) == _abi.ERR_UNSUPPORTED
    assert "no CUDA device" in moe.moe_nvfp4_last_error()


def test_forward_host_passes_the_callers_buffers(monkeypatch):
    """The binding hands the C entry point the caller's own host arrays (no copies when they
    are already contiguous and of the right type) and rejects an output it cannot fill."""
    calls = []

    class FakeLib:
        def moe_nvfp4_forward_host(self, x, lg, T, bank, k, out, stream):
            calls.append((x.value, lg.value, T, k, out.value, stream.value))
            return 0

    class Stream:
        cuda_stream = 1234

    monkeypatch.setattr(moe, "_LIB", FakeLib())
    x = np.zeros((3, 256), np.uint16)
    lg = np.zeros((3, 16), np.float32)
    out = np.empty_like(x)
    assert moe.moe_nvfp4_forward_host(x, lg, _bank(), 2, out_host=out, stream=Stream()) is out
    assert calls == [(x.ctypes.data, lg.ctypes.data, 3, 2, out.ctypes.data, 1234)]
    got = moe.moe_nvfp4_forward_host(x, lg.astype(np.float64), _bank(), 2, stream=Stream())
    assert got.shape == x.shape and got.dtype == np.uint16 and calls[-1][1] != lg.ctypes.data
    with pytest.raises(ValueError):
        moe.moe_nvfp4_forward_host(x, lg, _bank(), 2, out_host=np.empty((2, 256), np.uint16), stream=Stream())


# The Python binding checks tensors against the bank before calling the C library, which only
# sees raw pointers: a wrong width, dtype, layout or device would otherwise read or write out of
# bounds.  These run on the CPU: every check fires before any CUDA call.
def _cpu(shape, dtype):
    import torch
    return torch.zeros(shape, dtype=dtype)


@pytest.mark.parametrize("which,bad,msg", [
    ("x", ("shape", (4, 128)), "x has shape"),
    ("x", ("dtype", "float16"), "x has dtype"),
    ("logits", ("shape", (4, 15)), "logits has shape"),
    ("logits", ("dtype", "float64"), "logits has dtype"),
    ("out", ("shape", (3, 256)), "out has shape"),
    ("x", ("strided", None), "x must be contiguous"),
    ("x", ("cpu", None), "x must be on the current CUDA device"),
])
def test_binding_rejects_mismatched_tensors(which, bad, msg):
    import torch
    bank = _bank()
    t = dict(x=_cpu((4, 256), torch.bfloat16), logits=_cpu((4, 16), torch.float32), out=_cpu((4, 256), torch.bfloat16))
    kind, val = bad
    if kind == "shape":
        t[which] = _cpu(val, t[which].dtype)
    elif kind == "dtype":
        t[which] = _cpu(tuple(t[which].shape), getattr(torch, val))
    elif kind == "strided":
        t[which] = _cpu((256, 4), t[which].dtype).t()
    for fn in (lambda: moe.moe_nvfp4_forward(t["x"], t["logits"], bank, 2, out=t["out"]),
               lambda: moe.moe_nvfp4_forward_ex(t["x"], t["logits"], bank, 2, out=t["out"]),
               lambda: moe.moe_nvfp4_forward_noalloc(t["x"], t["logits"], bank, 2, out=t["out"])):
        with pytest.raises(ValueError, match=msg):
            fn()


def test_binding_rejects_mismatched_residual_and_route_inputs():
    import torch
    bank = _bank()
    x, lg, out = _cpu((4, 256), torch.bfloat16), _cpu((4, 16), torch.float32), _cpu((4, 256), torch.bfloat16)
    with pytest.raises(ValueError, match="x_next has shape"):
        moe.moe_nvfp4_forward_ex(x, lg, bank, 2, out=out, x_next=_cpu((4, 255), torch.bfloat16))
    with pytest.raises(ValueError, match="logits has dtype"):
        moe.moe_nvfp4_route(_cpu((4, 16), torch.float16), 2)
    with pytest.raises(ValueError, match="logits must be a 2-D"):
        moe.moe_nvfp4_route(_cpu((16,), torch.float32), 2)


def test_binding_rejects_mismatched_host_arrays():
    bank = _bank()
    x = np.zeros((4, 256), dtype=np.uint16)
    with pytest.raises(ValueError, match="x_host has shape"):
        moe.moe_nvfp4_forward_host(np.zeros((4, 128), dtype=np.uint16), np.zeros((4, 16), np.float32), bank, 2)
    with pytest.raises(ValueError, match="logits_host has shape"):
        moe.moe_nvfp4_forward_host(x, np.zeros((4, 17), np.float32), bank, 2)
    with pytest.raises(ValueError, match="out_host must be"):
        moe.moe_nvfp4_forward_host(x, np.zeros((4, 16), np.float32), bank, 2, out_host=np.zeros((4, 255), np.uint16))


def _enc(n=2, out_f=8, in_f=64, mode=0, w=0x20000, dst=0x40000, stride=4096, co=0, so=256, go=320):
    lib = moe.lib()
    return lib.moe_nvfp4_encode(ctypes.c_void_p(w), n, out_f, in_f, mode, ctypes.c_void_p(dst), stride, co, so, go,
                                None)


@pytest.mark.parametrize("kw", [dict(n=-1), dict(in_f=24), dict(in_f=0), dict(out_f=0), dict(mode=2),
                                dict(co=8), dict(stride=4008), dict(go=322), dict(so=16),    # codes overlap scales
                                dict(go=0), dict(stride=256, n=3)])                            # parts beyond the stride
def test_encode_rejects_bad_arguments_on_the_host(kw):
    assert _enc(**kw) == _abi.ERR_INVALID_ARG
    assert moe.moe_nvfp4_last_error() != ""


def test_encode_without_a_device_is_unsupported():
    assert _enc() == _abi.ERR_UNSUPPORTED
    assert moe.moe_nvfp4_last_launch_count() == 0


def _fwd_w4a4(bank, T=4, k=2, taps=None):
    lib = moe.lib()
    return lib.moe_nvfp4_forward_w4a4(ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), T, ctypes.byref(bank),
                                      ctypes.c_void_p(0x50000), k, ctypes.c_void_p(0x40000), None, None, 0, taps, None)


def test_w4a4_host_validation_runs_before_the_device():
    lib = moe.lib()
    assert _fwd_w4a4(_bank(), k=0) == _abi.ERR_INVALID_ARG
    assert _fwd_w4a4(_bank(), T=-1) == _abi.ERR_INVALID_ARG
    for H, I in ((384, 256), (256, 128)):
        lay = moe_inputs.record_layout(16, H, I)
        b = _bank(hidden=H, intermediate=I, record_stride=lay.record_stride, codes_off=lay.codes_off,
                  scales_off=lay.scales_off, global_off=lay.global_off)
        assert _fwd_w4a4(b) == _abi.ERR_UNSUPPORTED
        assert "W4A4 path needs H % 256 == 0 and I % 256 == 0" in lib.moe_nvfp4_last_error().decode()


def test_w4a4_binding_checks_scales_and_taps():
    import torch
    bank = _bank()
    x, lg, out = _cpu((4, 256), torch.bfloat16), _cpu((4, 16), torch.float32), _cpu((4, 256), torch.bfloat16)
    with pytest.raises(ValueError, match="act_scales has shape"):
        moe.moe_nvfp4_forward_w4a4(x, lg, bank, _cpu((16,), torch.float32), 2, out=out)
    with pytest.raises(ValueError, match="act_scales has dtype"):
        moe.moe_nvfp4_forward_w4a4(x, lg, bank, _cpu((16, 2), torch.float16), 2, out=out)


# ---- experts-only call and expert parallelism: host validation (nothing reaches a device)

def _vp(v):
    return ctypes.c_void_p(v)


def test_experts_call_rejects_bad_arguments_on_the_host():
    lib = moe.lib()
    b = _bank()
    call = lambda R=4, path=0, flags=0, bank=b: lib.moe_nvfp4_experts(        # noqa: E731
        _vp(0x20000), _vp(0x30000), R, ctypes.byref(bank) if bank is not None else None, _vp(0x40000), None, 0, path,
        flags, None)
    assert call(bank=None) == _abi.ERR_INVALID_ARG
    assert call(R=-1) == _abi.ERR_INVALID_ARG
    assert call(path=7) == _abi.ERR_INVALID_ARG
    assert call(flags=2) == _abi.ERR_INVALID_ARG
    assert "flags" in moe.moe_nvfp4_last_error()
    assert call(bank=_bank(hidden=200)) == _abi.ERR_UNSUPPORTED


def test_experts_workspace_bytes():
    f = moe.moe_nvfp4_experts_workspace_bytes
    assert f(-1, 16, 512, 256) == 0 and f(8, 0, 512, 256) == 0 and f(8, 16, 64, 256) == 0
    small, big = f(8, 16, 512, 256), f(4096, 16, 512, 256)
    assert 0 < small < big
    # the h and y regions alone: R x (I + H) x 4 bytes
    assert big >= 4096 * (256 + 512) * 4


@pytest.mark.parametrize("G,E,rank,layout,rows,code", [
    (0, 8, 0, 0, 0, _abi.ERR_INVALID_ARG),     # no ranks
    (65, 130, 0, 0, 0, _abi.ERR_INVALID_ARG),  # more ranks than the kernels take
    (3, 8, 0, 0, 0, _abi.ERR_INVALID_ARG),     # experts do not split evenly
    (2, 8, 2, 0, 0, _abi.ERR_INVALID_ARG),     # rank outside 0..G-1
    (2, 8, 0, 2, 0, _abi.ERR_INVALID_ARG),     # unknown layout
    (2, 8, 0, 0, -1, _abi.ERR_INVALID_ARG),    # negative row count
])
def test_ep_plan_rejects_bad_arguments(G, E, rank, layout, rows, code):
    lib = moe.lib()
    assert lib.moe_nvfp4_ep_plan(_vp(0x1000), G, E, rank, layout, _vp(0x2000), _vp(0x3000), rows, None) == code


def test_ep_dispatch_and_combine_reject_bad_arguments():
    lib = moe.lib()
    ptrs = (ctypes.c_void_p * 2)(0x50000, 0x60000)
    disp = lambda T=4, k=2, H=512, E=8, G=2, cap=16: lib.moe_nvfp4_ep_dispatch(     # noqa: E731
        _vp(0x20000), T, k, H, E, _vp(0x1000), _vp(0x2000), _vp(0x3000), _vp(0x4000), G, ptrs, cap, None)
    assert disp(k=0) == _abi.ERR_INVALID_ARG
    assert disp(k=9) == _abi.ERR_INVALID_ARG        # k > E
    assert disp(T=-1) == _abi.ERR_INVALID_ARG
    assert disp(E=9) == _abi.ERR_INVALID_ARG        # 9 experts over 2 ranks
    assert disp(H=12) == _abi.ERR_UNSUPPORTED       # not a multiple of 8
    assert disp(H=8200) == _abi.ERR_UNSUPPORTED     # above 8192
    comb = lambda T=4, k=2, H=512, E=8, G=2, cap=16: lib.moe_nvfp4_ep_combine(      # noqa: E731
        _vp(0x20000), T, k, H, E, _vp(0x1000), _vp(0x2000), _vp(0x3000), _vp(0x4000), _vp(0x5000), G, ptrs, cap,
        _vp(0x70000), None, None)
    assert comb(k=0) == _abi.ERR_INVALID_ARG
    assert comb(G=0) == _abi.ERR_INVALID_ARG
    assert comb(H=12) == _abi.ERR_UNSUPPORTED


def test_gather_rows_combine_and_buffers_reject_bad_arguments():
    lib = moe.lib()
    assert lib.moe_nvfp4_gather_rows(_vp(0x20000), _vp(0x1000), 4, 0, 512, _vp(0x30000), None) == _abi.ERR_INVALID_ARG
    assert lib.moe_nvfp4_gather_rows(_vp(0x20000), _vp(0x1000), 4, 2, 500, _vp(0x30000), None) == \
        _abi.ERR_UNSUPPORTED
    assert lib.moe_nvfp4_combine(_vp(0x1000), _vp(0x2000), _vp(0x3000), -1, 2, 512, None, _vp(0x4000), None,
                                 None) == _abi.ERR_INVALID_ARG
    p = ctypes.c_void_p()
    h = (ctypes.c_uint8 * 64)()
    assert lib.moe_nvfp4_ep_buffer_create(0, ctypes.byref(p), h) == _abi.ERR_INVALID_ARG
    assert lib.moe_nvfp4_ep_buffer_open(None, ctypes.byref(p)) == _abi.ERR_INVALID_ARG
    assert lib.moe_nvfp4_ep_buffer_close(None) == _abi.OK          # closing nothing is a no-op
    assert lib.moe_nvfp4_ep_buffer_destroy(None) == _abi.OK


def test_ep_bindings_check_tensors_before_devices():
    import torch
    b = _bank(num_experts=8, hidden=256)
    with pytest.raises(ValueError):          # ids of the wrong dtype
        moe.moe_nvfp4_experts(torch.zeros((4, 256), dtype=torch.bfloat16), torch.zeros(4, dtype=torch.int64), b)
    with pytest.raises(ValueError):          # y rows of the wrong width
        moe.moe_nvfp4_experts(torch.zeros((4, 256), dtype=torch.bfloat16), torch.zeros(4, dtype=torch.int32), b,
                              y_rows=torch.zeros((4, 128), dtype=torch.float32))
    with pytest.raises(ValueError):          # counts of the wrong dtype
        moe.moe_nvfp4_ep_plan(torch.zeros((2, 8), dtype=torch.int64), 0, 0)
    with pytest.raises(ValueError):          # perm of the wrong length
        moe.moe_nvfp4_gather_rows(torch.zeros((4, 256), dtype=torch.bfloat16), torch.zeros(7, dtype=torch.int32), 2,
                                  rows=torch.zeros((8, 256), dtype=torch.bfloat16))
    with pytest.raises(ValueError):          # an ep buffer handle has 64 bytes
        moe.moe_nvfp4_ep_buffer_open(b"short")
