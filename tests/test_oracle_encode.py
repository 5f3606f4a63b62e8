"""Pins of the oracle's NVFP4 encoder (BF16 weights -> E2M1 codes, E4M3 block scales, F32 global),
each against something other than the encoder itself: the ml_dtypes float4/float8 conversions
(library rounding routines), hand-derived ties (tests/golden/nvfp4_encode_ties.txt), exact
rational arithmetic, the oracle's independently pinned decoder, closed-form error bounds and
invariances of the format.

Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section "What this
pack holds" (the record, the g / 2688 convention); page "Running Beam-1.0 (501B) on workstation
GPUs" (data-free NVFP4A16 quantization of the experts)."""
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import moe_inputs
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "nvfp4_encode_ties.txt")


def _bf16(v):
    return moe_inputs.gen.to_bf16_bits(np.asarray(v, dtype=np.float32))


def _f(bits):
    return oracle.bf16_bits_to_f64(bits)


def test_e2m1_rounding_matches_ml_dtypes_on_a_dense_sweep():
    r = np.concatenate([np.linspace(-7.0, 7.0, 200001, dtype=np.float32),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)])
    got = oracle.E2M1_VALUES[oracle.e2m1_round(r)]
    want = r.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(got, want)


def test_e4m3_rounding_matches_ml_dtypes_below_the_saturation_point():
    # every E4M3 value, every midpoint between neighbours, and a random sweep, all below 464
    vals = oracle.E4M3_VALUES[:0x7F]
    mids = (vals[:-1] + vals[1:]) / 2
    rnd = np.random.default_rng(0).uniform(0, 463.9, 100000)
    v = np.concatenate([vals, mids, rnd]).astype(np.float32)
    got = oracle.E4M3_VALUES[oracle.e4m3_round(v)]
    want = v.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(got, want)
    # at and beyond 464 (where ml_dtypes gives NaN) the encoder saturates to 448
    assert np.all(oracle.e4m3_round(np.array([464.0, 480.0, 1e30], np.float32)) == 0x7E)


def test_hand_derived_ties():
    n = 0
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].split()
        if not line:
            continue
        kind, val, want = line[0], np.float32(line[1]), int(line[2])
        if line[1].startswith("-") and float(line[1]) == 0.0:
            val = np.float32(-0.0)
        fn = oracle.e2m1_round if kind == "e2m1" else oracle.e4m3_round
        assert int(fn(np.array([val], np.float32))[0]) == want, line
        n += 1
    assert n >= 30


def test_global_is_the_correctly_rounded_f32_of_amax_over_2688():
    rng = np.random.default_rng(1)
    for _ in range(200):
        w = _bf16(rng.standard_normal((4, 32)) * 2.0 ** rng.integers(-40, 40))
        amax, s2 = oracle.tensor_global(w)
        assert amax == np.abs(_f(w)).max()
        exact = Fraction(float(amax)) / 2688
        # s2 is an f32 and no f32 lies strictly closer to the exact quotient
        assert np.float32(s2) == s2
        up, dn = np.nextafter(s2, np.float32(np.inf)), np.nextafter(s2, np.float32(0))
        d = abs(Fraction(float(s2)) - exact)
        assert d <= abs(Fraction(float(up)) - exact) and d <= abs(Fraction(float(dn)) - exact)


def _representable(rng, out_f, in_f, s2_exp=-8):
    """BF16 weights that NVFP4 holds exactly: codes with one +-6 in every block, positive scale
    bytes, one block at the largest scale 448, global 2^s2_exp (then amax / 2688 = 2^s2_exp)."""
    nb = in_f // 16
    codes = rng.integers(0, 16, (out_f, nb, 16))
    pos = rng.integers(0, 16, (out_f, nb))
    sign = rng.integers(0, 2, (out_f, nb)) * 8
    np.put_along_axis(codes, pos[:, :, None], (7 + sign)[:, :, None], axis=2)
    scales = rng.integers(1, 0x7F, (out_f, nb)).astype(np.uint8)
    scales[0, 0] = 0x7E
    w = oracle.E2M1_VALUES[codes] * oracle.E4M3_VALUES[scales][:, :, None] * 2.0 ** s2_exp
    bits = _bf16(w.reshape(out_f, in_f))
    assert np.array_equal(_f(bits), w.reshape(out_f, in_f))         # exact in BF16
    return bits, codes.reshape(out_f, in_f).astype(np.uint8), scales


@pytest.mark.parametrize("mode", [0, 1])
def test_encoding_representable_weights_returns_their_codes_and_scales(mode):
    rng = np.random.default_rng(2)
    for s2e in (-8, -20, 3):
        bits, codes, scales = _representable(rng, 6, 64, s2e)
        c, s, g = oracle.encode_projection(bits, mode)
        # a -0 code (8) decodes to zero like code 0 and is encoded as +0 or -0 by its sign
        same = (c == codes) | ((codes & 7) == 0) & ((c & 7) == 0)
        assert same.all() and np.array_equal(s, scales)
        assert g == (np.float32(2.0 ** s2e) if mode == 0 else np.float32(2688.0 * 2.0 ** s2e))


def _decode(c, s, g, mode, in_f):
    return oracle.dequant(oracle.pack_codes(c), s, g, mode, in_f)


@pytest.mark.parametrize("dist", ["normal", "cauchy", "mixed"])
def test_every_weight_is_within_half_a_grid_step_of_its_code(dist):
    rng = np.random.default_rng(3)
    out_f, in_f = 32, 256
    if dist == "normal":
        w = rng.standard_normal((out_f, in_f))
    elif dist == "cauchy":
        w = rng.standard_cauchy((out_f, in_f))
    else:
        w = rng.standard_normal((out_f, in_f)) * 2.0 ** rng.integers(-20, 20, (out_f, 1))
    bits = _bf16(w)
    x = _f(bits)
    c, s, g = oracle.encode_projection(bits, 0)
    back = _decode(c, s, g, 0, in_f)
    eff = (oracle.E4M3_VALUES[s].astype(np.float32) * np.float32(g)).astype(np.float64)
    eff = np.repeat(eff, 16, axis=1)
    r = np.abs(x) / np.where(eff > 0, eff, 1)
    # spacing of the E2M1 grid around |w / eff| (0.5 up to 2, 1 up to 4, 2 above)
    gap = np.where(r <= 2, 0.5, np.where(r <= 4, 1.0, 2.0))
    err = np.abs(x - back)
    amax_b = np.repeat(np.max(np.abs(x).reshape(out_f, -1, 16), axis=2), 16, axis=1)
    sb = np.repeat(s, 16, axis=1)
    # A normal E4M3 block scale is within 2^-4 of amax_b / (6 s2), so |w / eff| <= 6 / (1 - 2^-4)
    # = 6.4 and a ratio above 6 is saturated by less than the top half-gap.  A subnormal scale
    # (byte < 8) rounds more coarsely: a ratio above 6 then saturates to exactly 6.
    assert (r[sb >= 8] <= 6.4).all()
    sat = (r > 6) & (sb < 8)
    assert np.array_equal(np.abs(back[sat]), 6 * eff[sat])
    ok = np.where(eff > 0, (err <= eff * gap / 2 * (1 + 1e-6)) | sat, err <= amax_b)
    assert ok.all()
    assert np.max(np.abs(x)) == pytest.approx(float(g) * 2688, rel=1e-6)


def test_power_of_two_scaling_changes_only_the_global():
    rng = np.random.default_rng(4)
    bits = _bf16(rng.standard_normal((8, 128)))
    c0, s0, g0 = oracle.encode_projection(bits, 0)
    for k in (-30, -1, 5, 40):
        c, s, g = oracle.encode_projection(_bf16(_f(bits) * 2.0 ** k), 0)
        assert np.array_equal(c, c0) and np.array_equal(s, s0) and g == np.float32(g0 * 2.0 ** k)


def test_block_scales_follow_their_16_inputs_and_rows():
    rng = np.random.default_rng(5)
    w = rng.uniform(-1, 1, (4, 64))
    w[2, 37] = 300.0                     # block (2, 2) holds the tensor's largest value
    w[1, 5] = 0.0
    w[1, :16] = 0.0                      # block (1, 0) is all zero
    bits = _bf16(w)
    c, s, g = oracle.encode_projection(bits, 0)
    assert s[2, 2] == 0x7E and s[1, 0] == 0 and (c[1, :16] & 7 == 0).all()
    assert np.count_nonzero(s == 0x7E) == 1
    perm = np.array([3, 0, 2, 1])
    cp, sp, gp = oracle.encode_projection(bits[perm], 0)
    assert np.array_equal(cp, c[perm]) and np.array_equal(sp, s[perm]) and gp == g


def test_tiny_blocks_and_zero_tensors():
    w = np.zeros((2, 32), np.float32)
    w[0, 0] = 1000.0
    w[1, 16:] = 1e-30                    # far below 2^-10 of the block scale unit: scale 0
    w[1, 17] = -1e-30
    c, s, g = oracle.encode_projection(_bf16(w), 0)
    assert s[1, 1] == 0 and (c[1, 16:] & 7 == 0).all() and c[1, 17] == 8
    c, s, g = oracle.encode_projection(_bf16(np.zeros((3, 16))), 1)
    assert g == 0 and not s.any() and not c.any()


def test_mode_one_stores_amax_and_reproduces_the_multiplier():
    rng = np.random.default_rng(6)
    bits = _bf16(rng.standard_normal((8, 64)) * 37.0)
    c0, s0, g0 = oracle.encode_projection(bits, 0)
    c1, s1, g1 = oracle.encode_projection(bits, 1)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    assert g1 == np.abs(_f(bits)).max()
    assert np.float32(oracle.global_multiplier(g1, 1)) == g0


def test_pack_codes_inverts_the_decoder():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 16, (5, 48)).astype(np.uint8)
    assert np.array_equal(oracle.decode_codes(oracle.pack_codes(codes), 48), codes)
