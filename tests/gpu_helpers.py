"""Helpers shared by the GPU parity tests: device banks, tensors, and the oracle's pool."""
import multiprocessing
import os

import numpy as np

import moe_inputs
from moe_inputs import device as mdev

_POOL = None


def oracle_pool():
    """A spawn-context process pool for the oracle (never forked after CUDA init)."""
    global _POOL
    if _POOL is None:
        n = max(1, min(32, (os.cpu_count() or 1)))
        _POOL = multiprocessing.get_context("spawn").Pool(n)
    return _POOL


def pool_map(fn, jobs):
    return oracle_pool().map(fn, list(jobs), chunksize=1)


def device_bank(cfg, layer=0, global_mode=0, seed=None):
    """(uint8 CUDA tensor, moe_nvfp4_bank) for one layer of cfg, written on the device."""
    import nvfp4_weight_only_top_b200 as moe
    lay = cfg.layout
    s = cfg.seed if seed is None else seed
    buf = mdev.bank_tensor(lay, s, layer, global_mode)
    bank = moe.make_bank(buf.data_ptr(), lay.E, lay.H, lay.I, lay.record_stride, lay.codes_off,
                         lay.scales_off, lay.global_off, global_mode)
    return buf, bank


def bf16_tensor(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bits_of(t) -> np.ndarray:
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
