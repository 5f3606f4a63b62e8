"""moe_nvfp4_forward_noalloc: the entry point for callers that cannot allocate device memory
(runtimes that reserve all device memory up front, latency-critical loops that cannot afford
an allocation's synchronisation).  It must give the same layer output as moe_nvfp4_forward,
call after call, although every call reuses one fixed scratch array inside the library.

This file is collected last on purpose: it must pass both on its own in a fresh process and
after every other test has run in the same process.
"""
import ctypes

import numpy as np
import pytest

import moe_inputs
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of, device_bank, pool_map

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "decode_t1", "decode_t64_zipf"])
def test_noalloc_matches_forward_on_two_calls_in_a_row(name):
    """The same kernels run in the same order on the same inputs, only the scratch differs: the
    outputs must be identical bit for bit on each of two calls in a row (the second reads a
    fixed array that still holds the first call's values), and within the layer tolerance of
    the FP64 oracle."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS[name]
    buf, bank = device_bank(cfg)
    lib = moe.lib()
    tokens = moe_inputs.sample_tokens(cfg.T, 64, cfg.seed)
    for call in range(2):                      # different inputs on each call
        xb = moe_inputs.make_x(cfg, seed=cfg.seed + call)
        lgn = moe_inputs.make_logits(cfg, seed=cfg.seed + call)
        x = bf16_tensor(xb)
        lg = torch.from_numpy(lgn).cuda()
        ref = moe.moe_nvfp4_forward(x, lg, bank, cfg.k)
        out = torch.empty_like(x)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = lib.moe_nvfp4_forward_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(lg.data_ptr()),
                                           x.shape[0], ctypes.byref(bank), cfg.k,
                                           ctypes.c_void_p(out.data_ptr()), stream)
        assert rc == 0, moe.moe_nvfp4_last_error()
        torch.cuda.synchronize()
        assert moe.moe_nvfp4_device_status() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{name} call {call}"
        src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I)
        want = oracle.layer_forward(xb, lgn, cfg.k, src, tokens=tokens, map_fn=pool_map)["out"]
        assert_layer_close(oracle.bf16_bits_to_f64(bits_of(out)[tokens]), want, f"{name} call {call} vs oracle")


def test_noalloc_rejects_scratch_beyond_its_array():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["decode_t1"]
    buf, bank = device_bank(cfg)
    T = 4096                                    # needs far more than the fixed array holds
    x = torch.zeros((T, cfg.H), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((T, cfg.E), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_nvfp4_forward_noalloc(x, lg, bank, cfg.k)
    assert ei.value.code == -4 and "fixed array" in str(ei.value)
    assert moe.moe_nvfp4_last_launch_count() == 0
