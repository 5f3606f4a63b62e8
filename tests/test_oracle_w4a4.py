"""Pins of the oracle's W4A4 variant (NVFP4 weights and NVFP4 activations), each against something
other than the code under test: an activation quantizer assembled from the ml_dtypes float4/float8
conversions (library rounding routines), numbers that are exactly representable, closed forms of
saturation and of power-of-two scaling, a brute-force tiny layer written out with plain loops,
and invariance under expert relabelling.

Page "Beam-1.0-501B-A23B, EXL3 3-bit ...", section "Fidelity": the official NVFP4 release served on
Blackwell with FP4 activations, against the weights-only build; page "Beam 1.0 501B-A23B,
streaming pack, NVFP4 experts / MLX 8-bit residents", section "What this pack holds": the release
carries activation scales (input_scale) that the BF16-activation build leaves unused.  The reading
pinned here: a routed row of expert e quantizes its token's activations with that expert's input
multiplier s_x[e] as the NVFP4 global, block scales and codes found from the values by the
encoder's rounding rule, and quantizes its f32 mid values with s_h[e] before the down
projection."""
import ml_dtypes
import numpy as np
import pytest

import moe_inputs
import oracle

F32 = np.float32


def _ml_quantize(v, s2):
    """Reference NVFP4 quantizer from library conversions: per block of 16, the block scale is
    float8_e4m3fn(f32(amax / f32(6 s2))) (clamped to 448 first: ml_dtypes has no saturating
    cast), each value is float4_e2m1fn(f32(v / f32(scale s2))) (clamped to +-6).  Returns the
    decoded FP64 values and the scale values."""
    v = np.asarray(v, F32)
    rows, n = v.shape
    s2 = np.broadcast_to(np.asarray(s2, F32).reshape(-1), (rows,))
    out = np.empty((rows, n))
    sc_out = np.empty((rows, n // 16))
    for r in range(rows):
        for b in range(n // 16):
            blk = v[r, 16 * b:16 * b + 16]
            q = F32(F32(np.max(np.abs(blk))) / F32(F32(6.0) * s2[r]))
            sc = np.array([min(q, F32(448.0))], F32).astype(ml_dtypes.float8_e4m3fn).astype(F32)[0]
            eff = F32(sc * s2[r])
            sc_out[r, b] = float(sc)
            if eff == 0:
                out[r, 16 * b:16 * b + 16] = 0.0
                continue
            t = np.clip((blk / eff).astype(F32), F32(-6.0), F32(6.0))
            e2 = t.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
            out[r, 16 * b:16 * b + 16] = e2 * float(sc) * float(s2[r])
    return out, sc_out


@pytest.mark.parametrize("seed", [0, 1])
def test_static_quantizer_matches_library_conversions(seed):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((6, 64)) * np.array([1e-3, 1.0, 30.0, 1.0, 5e3, 0.2])[:, None]).astype(F32)
    v[1, :16] = 0.0                                     # an all-zero block
    v[3, 16:32] *= 1e-6                                  # a block far below its row's multiplier
    s2 = np.array([1e-6, 3e-4, 1e-2, 4e-4, 2.0, 1e-4], F32)
    codes, scales, dec = oracle.quantize_static(v, s2)
    want, want_sc = _ml_quantize(v, s2)
    assert np.array_equal(dec, want)
    assert np.array_equal(oracle.E4M3_VALUES[scales], want_sc)
    assert np.array_equal(oracle.decode_blocks(codes, scales, s2), dec)


def test_static_quantizer_reproduces_representable_rows():
    rng = np.random.default_rng(2)
    rows, n = 4, 64
    s2 = np.array([2.0 ** -10, 3.0 * 2.0 ** -12, 0.125, 5.0 * 2.0 ** -16], F32)   # few mantissa bits
    sbytes = rng.integers(0x20, 0x70, size=(rows, n // 16)).astype(np.uint8)
    codes = rng.integers(0, 16, size=(rows, n)).astype(np.uint8)
    codes[:, ::16] = 7                                    # each block's largest magnitude is 6
    v64 = oracle.decode_blocks(codes, sbytes, s2)
    v = v64.astype(F32)
    assert np.array_equal(v.astype(np.float64), v64)     # exact in f32
    c2, s2b, dec = oracle.quantize_static(v, s2)
    assert np.array_equal(dec, v64)
    assert np.array_equal(s2b, sbytes)
    nz = oracle.E2M1_VALUES[codes] != 0
    assert np.array_equal(c2[nz], codes[nz])


def test_static_quantizer_saturates_at_6_x_448_x_multiplier():
    s2 = F32(1.0 / 64)
    v = np.array([[1e4, -1e4, 3e3, -2.7e3] * 4], F32)
    codes, scales, dec = oracle.quantize_static(v, s2)
    assert np.all(scales == 0x7E)                         # 448
    assert np.array_equal(dec[0], np.sign(v[0]) * 2688.0 / 64)


def test_static_quantizer_power_of_two_invariance():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((3, 48)).astype(F32)
    s2 = np.array([0.01, 0.003, 0.2], F32)
    c0, sc0, d0 = oracle.quantize_static(v, s2)
    for k in (-7, 5):
        c1, sc1, d1 = oracle.quantize_static(np.ldexp(v, k), np.ldexp(s2, k))
        assert np.array_equal(c0, c1) and np.array_equal(sc0, sc1)
        assert np.array_equal(np.ldexp(d0, k), d1)


def test_static_quantizer_uses_each_rows_own_multiplier():
    v = np.ones((2, 16), F32)
    _, _, d = oracle.quantize_static(v, np.array([1.0, 1.0 / 4096], F32))
    want, _ = _ml_quantize(v, np.array([1.0, 1.0 / 4096], F32))
    assert np.array_equal(d, want)
    assert d[0, 0] != d[1, 0]


def _brute_force_layer(x_bits, logits, k, mats, act_scales):
    """out [T, H] of the W4A4 layer, written with plain loops over tokens, slots, rows and
    columns; quantization by _ml_quantize; routing by sorting each token's logits (ties to the
    lower index) and a softmax over the k selected."""
    x = oracle.bf16_bits_to_f64(x_bits)
    T, H = x.shape
    out = np.zeros((T, H))
    for t in range(T):
        order = sorted(range(logits.shape[1]), key=lambda e: (-float(logits[t, e]), e))[:k]
        sel = np.array([float(logits[t, e]) for e in order])
        w = np.exp(sel - sel.max())
        w /= w.sum()
        for j, e in enumerate(order):
            Wg, Wu, Wd = mats[e]
            xq, _ = _ml_quantize(x[t:t + 1].astype(F32), act_scales[e, 0])
            I = Wg.shape[0]
            h = np.zeros(I, F32)
            for i in range(I):
                g = sum(Wg[i, c] * xq[0, c] for c in range(H))
                u = sum(Wu[i, c] * xq[0, c] for c in range(H))
                h[i] = F32(g / (1.0 + np.exp(-g)) * u)
            hq, _ = _ml_quantize(h[None, :], act_scales[e, 1])
            for c in range(H):
                out[t, c] += w[j] * sum(Wd[c, i] * hq[0, i] for i in range(I))
    return out


def _tiny(E=4, H=32, I=32, T=3, seed=5):
    cfg = moe_inputs.LayerConfig(name="tiny-w4a4", E=E, k=2, H=H, I=I, T=T, seed=seed)
    mats = [oracle.GeneratedRecords(seed, 0, E, H, I)(e) for e in range(E)]
    x = moe_inputs.make_x(cfg)
    lg = moe_inputs.make_logits(cfg)
    # different multipliers per expert and per input, around 1/2688 of the inputs' typical maxima
    act = np.array([[3.0 / 2688 * (1 + e), 0.05 / 2688 * (2 + e)] for e in range(E)], F32)
    return cfg, x, lg, mats, act


def test_w4a4_layer_matches_brute_force_loops():
    cfg, x, lg, mats, act = _tiny()
    res = oracle.layer_forward(x, lg, cfg.k, lambda e: mats[e], act_scales=act)
    want = _brute_force_layer(x, lg, cfg.k, mats, act)
    assert np.max(np.abs(res["out"] - want)) <= 1e-9 * np.max(np.abs(want))
    # and it is not the BF16-activation layer
    a16 = oracle.layer_forward(x, lg, cfg.k, lambda e: mats[e])
    assert np.max(np.abs(a16["out"] - want)) > 1e-4 * np.max(np.abs(want))


def test_w4a4_layer_is_invariant_under_expert_relabelling():
    cfg, x, lg, mats, act = _tiny(E=5, seed=7)
    perm = np.array([3, 0, 4, 1, 2])              # new expert p holds old expert perm[p]
    a = oracle.layer_forward(x, lg, cfg.k, lambda e: mats[e], act_scales=act)
    b = oracle.layer_forward(x, lg[:, perm], cfg.k, lambda e: mats[perm[e]], act_scales=act[perm])
    assert np.max(np.abs(a["out"] - b["out"])) <= 1e-12 * np.max(np.abs(a["out"]))


def test_w4a4_teacher_forcing_reproduces_the_layer():
    cfg, x, lg, mats, act = _tiny(seed=9)
    a = oracle.layer_forward(x, lg, cfg.k, lambda e: mats[e], act_scales=act)
    b = oracle.layer_forward(x, lg, cfg.k, lambda e: mats[e], act_scales=act, h_rows=a["h"])
    assert np.array_equal(a["out"], b["out"])
    # a forced h that differs changes the result
    c = oracle.layer_forward(x, lg, cfg.k, lambda e: mats[e], act_scales=act, h_rows=a["h"] * F32(2.0))
    assert not np.array_equal(a["out"], c["out"])
