"""Small cases for ncu captures: a few layer calls on a bank that still exceeds L2.

    python -m nvfp4_weight_only_top_b200.ncu_case --case decode_t1_e16 --calls 4

Cases (full-size records H=5120, I=2560, only 16 experts resident = 354 MB > 126 MB L2):
  decode_t1_e16   T=1,  k=8, each call routes to 8 experts not used by the previous call
  decode_t16_e16  T=16, k=8
  decode_t64_e16  T=64, k=8
Every call is plain (no CUDA graph) on one stream; the process synchronises at the end.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

CASES = {"decode_t1_e16": (1, "decode"), "decode_t16_e16": (16, "decode"), "decode_t64_e16": (64, "decode"),
         "prefill_t4096_e16": (4096, "prefill")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", default="decode_t1_e16", choices=list(CASES))
    ap.add_argument("--calls", type=int, default=4)
    a = ap.parse_args()
    import torch
    import moe_inputs
    from moe_inputs import device as mdev
    import nvfp4_weight_only_top_b200 as moe
    T, path = CASES[a.case]
    E, k, H, I = 16, 8, 5120, 2560
    lay = moe_inputs.record_layout(E, H, I)
    buf = mdev.bank_tensor(lay, 0, 0)
    bank = moe.make_bank(buf.data_ptr(), E, H, I, lay.record_stride, lay.codes_off, lay.scales_off,
                         lay.global_off, 0)
    cfg = moe_inputs.LayerConfig(a.case, E, k, H, I, T)
    x = torch.from_numpy(moe_inputs.make_x(cfg).view(np.int16)).view(torch.bfloat16).cuda()
    if T == 1:
        lg = torch.from_numpy(moe_inputs.disjoint_routing_logits(E, k, a.calls, 2)).cuda()
    else:
        lg = torch.from_numpy(np.stack([moe_inputs.make_logits(cfg, layer=i) for i in range(a.calls)])).cuda()
    p = moe.PATH_DECODE if path == "decode" else moe.PATH_PREFILL
    for i in range(a.calls):
        moe.moe_nvfp4_forward_ex(x, lg[i], bank, k, path=p)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    print(f"{a.case}: {a.calls} calls ok")


if __name__ == "__main__":
    main()
