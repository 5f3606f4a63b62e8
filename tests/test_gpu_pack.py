"""Streaming packs on the GPU: a layer loaded from experts.bin is byte-identical to the generator's
bank and gives the same layer output; the integrity check stops a load at a corrupted record; and
the expert-row cache (a bounded set of record slots fed from the pack as the router selects
experts) reproduces the full layer bit for bit while it loads, hits and evicts.

Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", sections "What this
pack holds" (records, manifest, sha256, 4 KiB alignment, g / 2688 globals) and "How to run" (the
expert rows the GPU keeps per routed layer)."""
import os

import numpy as np
import pytest

import moe_inputs
from moe_inputs import pack as mpack
from moe_inputs import device as mdev
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of, pool_map

pytestmark = pytest.mark.gpu

E, H, I, LAYERS, SEED = 16, 1024, 512, 3, 4


@pytest.fixture(scope="module")
def pack_dir(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("gpu_pack"))
    mpack.write_pack(d, layers=LAYERS, E=E, H=H, I=I, seed=SEED)
    return d


def _full_bank(layer):
    import nvfp4_weight_only_top_b200 as moe
    lay = moe_inputs.record_layout(E, H, I)
    buf = mdev.bank_tensor(lay, SEED, layer, global_mode=1)
    return buf, moe.make_bank(buf.data_ptr(), E, H, I, lay.record_stride, lay.codes_off, lay.scales_off,
                              lay.global_off, 1)


def test_loaded_layer_equals_the_generated_bank(pack_dir):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    p = moe.Pack(os.path.join(pack_dir, "expert-manifest.json"))
    for layer in range(LAYERS):
        buf, bank = p.load_bank(layer, verify=True)
        ref, rbank = _full_bank(layer)
        torch.cuda.synchronize()
        lay = moe_inputs.record_layout(E, H, I)
        a = buf.view(E, lay.record_stride)[:, :lay.record_bytes]
        b = ref.view(E, lay.record_stride)[:, :lay.record_bytes]
        assert torch.equal(a, b), f"layer {layer}"
        cfg = moe_inputs.LayerConfig("pack", E, 4, H, I, 5, 1, "normal", seed=layer)
        x = bf16_tensor(moe_inputs.make_x(cfg))
        lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()
        o1 = moe.moe_nvfp4_forward(x, lg, bank, 4)
        o2 = moe.moe_nvfp4_forward(x, lg, rbank, 4)
        torch.cuda.synchronize()
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    # a subset of experts into a caller-chosen stride
    dst = torch.zeros(3 * 2 ** 21, dtype=torch.uint8, device="cuda")
    p.load(1, dst, experts=[7, 0, 15], dst_stride=2 ** 21)
    torch.cuda.synchronize()
    for i, e in enumerate([7, 0, 15]):
        got = dst[i * 2 ** 21:i * 2 ** 21 + p.info["record_bytes"]].cpu().numpy()
        assert np.array_equal(got, mpack.pack_record(pack_dir, 1, e))
    p.close()


def test_verified_load_stops_at_a_corrupted_record(tmp_path):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    mpack.write_pack(str(tmp_path), layers=1, E=4, H=256, I=128, seed=2, corrupt=[(0, 2)])
    p = moe.Pack(str(tmp_path / "expert-manifest.json"))
    dst = torch.empty(4 * p.info["record_stride"], dtype=torch.uint8, device="cuda")
    p.load(0, dst, experts=[0, 1, 3])                 # intact records load
    with pytest.raises(moe.MoeError) as ei:
        p.load(0, dst, verify=True)
    assert ei.value.code == -7 and "expert 2" in str(ei.value)
    torch.cuda.synchronize()
    p.close()


def _logits_selecting(rng, T, k, experts):
    """[T, E] logits whose top k of each token are the given experts (rows of `experts`)."""
    lg = rng.standard_normal((T, E)).astype(np.float32)
    for t in range(T):
        lg[t, experts[t]] = 5.0 + rng.random(k).astype(np.float32)
    return lg


def test_rows_reproduce_the_full_layer_while_loading_and_evicting(pack_dir):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    p = moe.Pack(os.path.join(pack_dir, "expert-manifest.json"))
    layer, k, S = 2, 2, 6
    rows = moe.Rows(p, layer, S)
    buf, bank = _full_bank(layer)
    rng = np.random.default_rng(0)
    seen = set()
    calls = [(1, [[0, 1]]), (1, [[1, 2]]), (3, [[3, 4], [5, 0], [4, 5]]), (1, [[6, 7]]),
             (3, [[8, 9], [10, 11], [9, 8]]), (1, [[0, 11]]), (3, [[12, 13], [13, 14], [15, 12]])]
    for T, sel in calls:
        lg = _logits_selecting(rng, T, k, sel)
        x = bf16_tensor(moe_inputs.gen.to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32)))
        lgd = torch.from_numpy(lg).cuda()
        got = rows.forward(x, lgd, k)
        want = moe.moe_nvfp4_forward(x, lgd, bank, k)
        torch.cuda.synchronize()
        assert moe.moe_nvfp4_device_status() == 0
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), sel
        seen |= {e for s in sel for e in s}
    st = rows.stats()
    assert st["misses"] + st["hits"] == sum(len({e for s in sel for e in s}) for _, sel in calls)
    assert st["misses"] >= len(seen) and st["bytes_loaded"] == st["misses"] * p.info["record_bytes"]
    assert st["hits"] >= 1                                # expert 0, 1, 11 ... come back
    # the layer against the oracle once more, through the rows
    T = 3
    lg = _logits_selecting(rng, T, k, [[2, 3], [3, 14], [7, 2]])
    xb = moe_inputs.gen.to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    got = rows.forward(bf16_tensor(xb), torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    ref = oracle.layer_forward(xb, lg, k, oracle.GeneratedRecords(SEED, layer, E, H, I, 1), map_fn=pool_map)["out"]
    assert_layer_close(oracle.bf16_bits_to_f64(bits_of(got)), ref, "rows vs oracle")
    # a call selecting more experts than there are slots is refused
    lg = _logits_selecting(rng, 4, k, [[0, 1], [2, 3], [4, 5], [6, 7]])
    with pytest.raises(moe.MoeError) as ei:
        rows.forward(bf16_tensor(moe_inputs.gen.to_bf16_bits(np.zeros((4, H), np.float32))),
                     torch.from_numpy(lg).cuda(), k)
    assert ei.value.code == -2 and "row cache holds 6" in str(ei.value)
    rows.destroy()
    p.close()
