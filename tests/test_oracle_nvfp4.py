"""Pins of the oracle's NVFP4 decoding (CPU only).

The decoders are checked against library decodings (ml_dtypes, torch), the record geometry
against the numbers the streaming-pack page prints, and the index conventions against a
test-side encoder that writes known matrices in the stated layout.
"""

import ml_dtypes
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from conftest import load_golden


def test_e2m1_matches_ml_dtypes():
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = oracle.E2M1_VALUES
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))       # code 8 is -0.0


def test_e4m3_matches_torch_and_ml_dtypes():
    b = np.arange(256, dtype=np.uint8)
    ref_t = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref_m = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = oracle.E4M3_VALUES
    nan = np.isnan(ref_t)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2         # 0x7F and 0xFF only
    assert np.array_equal(got[~nan], ref_t[~nan])
    assert np.array_equal(got[~nan], ref_m[~nan])


def test_product_table_exact_and_2688():
    g = load_golden("record_geometry.txt")
    e2 = oracle.E2M1_VALUES
    e4 = oracle.E4M3_VALUES[~np.isnan(oracle.E4M3_VALUES)]
    # Every e2m1 x e4m3 product is exact in FP64 and in FP16/BF16 (6 significant bits).
    prod = np.outer(e2, e4)
    assert np.array_equal(prod.astype(np.float16).astype(np.float64), prod)
    assert np.array_equal(prod.astype(ml_dtypes.bfloat16).astype(np.float64), prod)
    # The page's denominator 2688 is the largest E2M1 magnitude times the largest finite E4M3.
    assert np.abs(e2).max() * np.abs(e4).max() == g["global_denominator"]


def test_record_geometry_matches_page():
    g = load_golden("record_geometry.txt")
    s = load_golden("layer_shape.txt")
    H, I = s["hidden"], s["intermediate"]
    # gate [I, H], up [I, H], down [H, I]
    rec = oracle.projection_bytes(I, H) * 2 + oracle.projection_bytes(H, I)
    assert rec == g["record_bytes"]
    stride = -(-rec // g["stride_alignment"]) * g["stride_alignment"]
    assert stride == g["record_stride"]
    assert g["routed_layers"] * g["experts"] == g["records"]
    assert g["routed_layers"] * stride == g["row_bytes"]
    assert g["records"] * 3 == g["projections"]
    assert s["down_mid_bytes"] == g["active_experts"] * I * 2
    lay = moe_inputs.record_layout(256, H, I)
    assert lay.record_bytes == g["record_bytes"] and lay.record_stride == g["record_stride"]
    # H * I is the only product that gives the page's record size.
    assert (g["record_bytes"] - 12) * 16 % (3 * 9) == 0
    assert (g["record_bytes"] - 12) * 16 // (3 * 9) == H * I


def _encode(W_codes: np.ndarray, S_bytes: np.ndarray):
    """Test-side writer of the stated layout: element (o, i) -> nibble i%8 of word i//8."""
    O, K = W_codes.shape
    words = np.zeros((O, K // 8), dtype=np.uint64)
    for i in range(K):
        words[:, i // 8] |= W_codes[:, i].astype(np.uint64) << np.uint64(4 * (i % 8))
    return words.astype('<u4'), S_bytes.astype(np.uint8)


def test_dequant_index_conventions():
    rng = np.random.default_rng(7)
    O, K = 6, 64
    codes = rng.integers(0, 16, (O, K))
    sbytes = rng.integers(0x18, 0x49, (O, K // 16))
    words, scales = _encode(codes, sbytes)
    W = oracle.dequant(words, scales, np.float32(0.25), 0, K)
    # brute force per element, via the library decoders
    e2 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    e4 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for o in range(O):
        for i in range(K):
            assert W[o, i] == e2[codes[o, i]] * e4[sbytes[o, i // 16]] * 0.25


def test_single_nibble_lands_in_its_column():
    O, K = 3, 32
    for o in range(O):
        for i in range(K):
            words = np.zeros((O, K // 8), dtype='<u4')
            words[o, i // 8] = np.uint32(2) << np.uint32(4 * (i % 8))      # code 2 = 1.0
            scales = np.full((O, K // 16), 0x38, dtype=np.uint8)               # 1.0
            W = oracle.dequant(words, scales, np.float32(1.0), 0, K)
            nz = np.argwhere(W != 0)
            assert nz.tolist() == [[o, i]] and W[o, i] == 1.0


def test_global_mode_1_is_f32_division():
    from fractions import Fraction
    for g in [np.float32(2688.0), np.float32(1.0), np.float32(0.0023292375 * 2688), np.float32(7.0),
              np.float32(1e-3), np.float32(3.0e4)]:
        m = oracle.global_multiplier(g, 1)
        exact = Fraction(float(g)) / 2688
        # an f32 value, and the correctly rounded one: no other f32 lies closer to g / 2688
        assert float(np.float32(m)) == m
        lo, hi = np.nextafter(np.float32(m), np.float32(-np.inf)), np.nextafter(np.float32(m), np.float32(np.inf))
        d = abs(Fraction(m) - exact)
        assert d <= abs(Fraction(float(lo)) - exact) and d <= abs(Fraction(float(hi)) - exact)
    assert oracle.global_multiplier(np.float32(2688.0), 1) == 1.0
    assert oracle.global_multiplier(np.float32(0.75), 0) == 0.75


def test_read_record_uses_descriptor_offsets():
    lay = moe_inputs.record_layout(4, 32, 16)
    rec = moe_inputs.record_bytes(3, 0, 1, lay)
    Wg, Wu, Wd = oracle.read_record(rec, 32, 16, lay.codes_off, lay.scales_off, lay.global_off)
    assert Wg.shape == (16, 32) and Wu.shape == (16, 32) and Wd.shape == (32, 16)
    gl = float(moe_inputs.global_value(32))
    # All scale bytes lie in 0x18..0x48, so every |weight| / global is an e2m1 x [2^-4, 4] product.
    for W in (Wg, Wu, Wd):
        r = np.abs(W) / gl
        assert r.max() <= 24.0 and (r[r > 0].min() >= 0.5 * 2 ** -4)
    # gate and up come from different parts of the record
    assert not np.array_equal(Wg, Wu)


def test_generator_scale_bytes_uniform_over_49_codes():
    lay = moe_inputs.record_layout(1, 256, 128)
    rec = moe_inputs.record_bytes(0, 0, 0, lay)
    sc = rec[lay.scales_off[0]:lay.global_off[0]]
    vals, cnt = np.unique(sc, return_counts=True)
    assert vals.min() == 0x18 and vals.max() == 0x48 and len(vals) == 49
    assert cnt.min() > 0.6 * cnt.mean()


@pytest.mark.parametrize("H,I", [(256, 128), (5120, 2560)])
def test_generator_codes_cover_16_values(H, I):
    lay = moe_inputs.record_layout(1, H, I)
    rec = moe_inputs.record_bytes(1, 2, 3, lay)
    b = rec[:lay.scales_off[0]]
    nib = np.concatenate([b & 15, b >> 4])
    cnt = np.bincount(nib, minlength=16)
    assert cnt.min() > 0.9 * cnt.mean()


def test_read_record_part_roles():
    """A hand-built record whose three projections hold different constants."""
    H, I = 32, 16
    lay = moe_inputs.record_layout(1, H, I)
    rec = np.zeros(lay.record_bytes, dtype=np.uint8)
    fills = {0: 0x22, 1: 0x44, 2: 0x66}             # codes 2 (1.0), 4 (2.0), 6 (4.0)
    for p, b in fills.items():
        n = I * H // 2
        rec[lay.codes_off[p]:lay.codes_off[p] + n] = b
        rec[lay.scales_off[p]:lay.scales_off[p] + I * H // 16] = 0x38 + 8 * p   # 1, 2, 4
        rec[lay.global_off[p]:lay.global_off[p] + 4] = np.array([0.5 * (p + 1)], '<f4').view(np.uint8)
    Wg, Wu, Wd = oracle.read_record(rec, H, I, lay.codes_off, lay.scales_off, lay.global_off)
    assert Wg.shape == (I, H) and np.all(Wg == 1.0 * 1.0 * 0.5)
    assert Wu.shape == (I, H) and np.all(Wu == 2.0 * 2.0 * 1.0)
    assert Wd.shape == (H, I) and np.all(Wd == 4.0 * 4.0 * 1.5)


def test_decode_codes_inverts_the_writer():
    rng = np.random.default_rng(17)
    codes = rng.integers(0, 16, (5, 48))
    words, _ = _encode(codes, np.zeros((5, 3)))
    assert np.array_equal(oracle.decode_codes(words, 48), codes)


@pytest.mark.parametrize("part", [0, 1, 2])
def test_read_record_index_layout_of_each_part(part):
    """Per projection of a hand-built record: one nonzero code lands at its (out, in) position,
    and one distinct block scale covers exactly its 16 inputs of its row (gate and up are
    [I, H], down is [H, I])."""
    H, I = 64, 32
    lay = moe_inputs.record_layout(1, H, I)
    O, K = [(I, H), (I, H), (H, I)][part]
    rng = np.random.default_rng(23 + part)
    for o, i in [(0, 0), (O - 1, K - 1), (1, K - 9), (O - 2, 17)] + [tuple(v) for v in rng.integers(0, [O, K], (4, 2))]:
        rec = np.zeros(lay.record_bytes, dtype=np.uint8)
        for p in range(3):
            rec[lay.scales_off[p]:lay.scales_off[p] + O * K // 16] = 0x38          # 1.0
            rec[lay.global_off[p]:lay.global_off[p] + 4] = np.array([1.0], '<f4').view(np.uint8)
        byte = lay.codes_off[part] + (o * K + i) // 2
        rec[byte] = 0x2 << (4 * (i % 2))                                          # code 2 = 1.0
        W = oracle.read_record(rec, H, I, lay.codes_off, lay.scales_off, lay.global_off)
        assert np.argwhere(W[part] != 0).tolist() == [[o, i]] and W[part][o, i] == 1.0
        assert all(not np.any(W[q]) for q in range(3) if q != part)
    for o, b in [(0, 0), (O - 1, K // 16 - 1), (O // 2, 1)]:
        rec = np.zeros(lay.record_bytes, dtype=np.uint8)
        rec[lay.codes_off[part]:lay.codes_off[part] + O * K // 2] = 0x22              # all 1.0
        rec[lay.scales_off[part]:lay.scales_off[part] + O * K // 16] = 0x38
        rec[lay.scales_off[part] + o * (K // 16) + b] = 0x40                         # 2.0
        rec[lay.global_off[part]:lay.global_off[part] + 4] = np.array([1.0], '<f4').view(np.uint8)
        W = oracle.read_record(rec, H, I, lay.codes_off, lay.scales_off, lay.global_off)[part]
        want = np.ones((O, K))
        want[o, 16 * b:16 * b + 16] = 2.0
        assert np.array_equal(W, want)
