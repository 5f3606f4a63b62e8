"""The W4A4 layer (NVFP4 activations on tcgen05 kind::mxf4nvf4) against the FP64 oracle.

Every integer the path decides is compared bit for bit, with the decision taken on the same f32
value on both sides: the codes and block scales of each routed slot's quantized x (from the exact
BF16 input), and those of its quantized mid values (the oracle quantizes the f32 h that the GPU
formed, read back through the taps).  The f32 mid values themselves, and the layer's output with
the GPU's h fed to the oracle (teacher forcing), are compared within the layer tolerance; the
output without teacher forcing too."""
import numpy as np
import pytest

import moe_inputs
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of, device_bank, pool_map

pytestmark = pytest.mark.gpu


def _packed(codes):
    """Oracle codes [n, m] (one per byte) -> bytes [n, m/2], lower index in the low nibble."""
    return oracle.pack_codes(codes).view(np.uint8).reshape(codes.shape[0], -1)


def _run(cfg, bank, xb, lg, act, taps=True):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    R, H, I = cfg.T * cfg.k, cfg.H, cfg.I
    x = bf16_tensor(xb)
    logits = torch.from_numpy(lg).cuda()
    a = torch.from_numpy(act).cuda()
    t = {}
    if taps:
        t = {"x_codes": torch.zeros((R, H // 2), dtype=torch.uint8, device="cuda"),
             "x_scales": torch.zeros((R, H // 16), dtype=torch.uint8, device="cuda"),
             "h": torch.zeros((R, I), dtype=torch.float32, device="cuda"),
             "h_codes": torch.zeros((R, I // 2), dtype=torch.uint8, device="cuda"),
             "h_scales": torch.zeros((R, I // 16), dtype=torch.uint8, device="cuda")}
    out = moe.moe_nvfp4_forward_w4a4(x, logits, bank, a, cfg.k, taps=t)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    return bits_of(out), {kk: v.cpu().numpy() for kk, v in t.items()}


def _check_slots(cfg, xb, lg, act, taps, slots):
    """Bit-exact checks of the quantized x and of the quantization of the GPU's h, per slot."""
    ids, _ = oracle.route(lg, cfg.k)
    x = oracle.bf16_bits_to_f64(xb).astype(np.float32)
    for r in slots:
        t, j = divmod(int(r), cfg.k)
        e = int(ids[t, j])
        c, s, _ = oracle.quantize_static(x[t:t + 1], act[e, 0])
        assert np.array_equal(taps["x_codes"][r], _packed(c)[0]), f"x codes of slot {r}"
        assert np.array_equal(taps["x_scales"][r], s[0]), f"x scales of slot {r}"
        c, s, _ = oracle.quantize_static(taps["h"][r:r + 1], act[e, 1])
        assert np.array_equal(taps["h_codes"][r], _packed(c)[0]), f"h codes of slot {r}"
        assert np.array_equal(taps["h_scales"][r], s[0]), f"h scales of slot {r}"


def _layer_check(cfg, xb, lg, act, out, taps, tokens, what):
    src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I)
    h_gpu = taps["h"].reshape(cfg.T, cfg.k, cfg.I)
    ref = oracle.layer_forward(xb, lg, cfg.k, src, tokens=tokens, map_fn=pool_map, act_scales=act)
    # mid values: the GPU's f32 h against the oracle's (from the same quantized x)
    assert_layer_close(h_gpu[ref["tokens"]].reshape(-1, cfg.I), ref["h"].reshape(-1, cfg.I), f"{what} h")
    forced = oracle.layer_forward(xb, lg, cfg.k, src, tokens=tokens, map_fn=pool_map, act_scales=act, h_rows=h_gpu)
    got = oracle.bf16_bits_to_f64(out[ref["tokens"]])
    assert_layer_close(got, forced["out"], f"{what} teacher-forced")
    assert_layer_close(got, ref["out"], f"{what} free-running")


@pytest.mark.parametrize("E,k,H,I,T", [(16, 2, 512, 256, 8), (16, 4, 512, 512, 1), (64, 4, 1024, 512, 40),
                                       (8, 8, 768, 256, 70), (32, 8, 1024, 768, 300)])
def test_w4a4_small_layers(E, k, H, I, T):
    cfg = moe_inputs.LayerConfig(name=f"w4a4_{E}_{k}_{H}_{I}_{T}", E=E, k=k, H=H, I=I, T=T, seed=11)
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    act = moe_inputs.make_act_scales(E, seed=cfg.seed)
    out, taps = _run(cfg, bank, xb, lg, act)
    _check_slots(cfg, xb, lg, act, taps, range(T * k))
    _layer_check(cfg, xb, lg, act, out, taps, None, cfg.name)


def test_w4a4_full_prefill_sampled():
    cfg = moe_inputs.CONFIGS["prefill_t8192"]
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    act = moe_inputs.make_act_scales(cfg.E, seed=cfg.seed)
    out, taps = _run(cfg, bank, xb, lg, act)
    tokens = moe_inputs.sample_tokens(cfg.T, 512, cfg.seed)
    slots = (tokens[:64, None] * cfg.k + np.arange(cfg.k)[None, :]).reshape(-1)
    _check_slots(cfg, xb, lg, act, taps, slots)
    _layer_check(cfg, xb, lg, act, out, taps, tokens, "prefill_t8192 w4a4")


def test_w4a4_taps_do_not_change_the_result_and_repeat_bitwise():
    cfg = moe_inputs.LayerConfig(name="w4a4_rep", E=32, k=4, H=1024, I=512, T=200, seed=3)
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    act = moe_inputs.make_act_scales(cfg.E, seed=cfg.seed)
    a, _ = _run(cfg, bank, xb, lg, act, taps=True)
    b, _ = _run(cfg, bank, xb, lg, act, taps=False)
    c, _ = _run(cfg, bank, xb, lg, act, taps=False)
    assert np.array_equal(a, b) and np.array_equal(b, c)


def test_w4a4_saturating_and_tiny_multipliers():
    """Multipliers far below the data (most values saturate at 6 x 448 x s) and far above it
    (most blocks get small or zero scales): still bit-exact decisions and the layer tolerance."""
    cfg = moe_inputs.LayerConfig(name="w4a4_sat", E=16, k=2, H=512, I=256, T=24, seed=5)
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    act = moe_inputs.make_act_scales(cfg.E, seed=cfg.seed)
    act[::2] *= np.float32(1.0 / 64)
    act[1::2] *= np.float32(2.0 ** 20)
    out, taps = _run(cfg, bank, xb, lg, act)
    _check_slots(cfg, xb, lg, act, taps, range(cfg.T * cfg.k))
    _layer_check(cfg, xb, lg, act, out, taps, None, "w4a4 saturating")


def test_w4a4_rejects_unsupported_shapes_and_bad_taps():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.LayerConfig(name="w4a4_bad", E=16, k=2, H=384, I=256, T=4, seed=1)
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()
    act = torch.from_numpy(moe_inputs.make_act_scales(cfg.E)).cuda()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_nvfp4_forward_w4a4(x, lg, bank, act, cfg.k)
    assert ei.value.code == -2
    cfg = moe_inputs.LayerConfig(name="w4a4_bad2", E=16, k=2, H=512, I=256, T=4, seed=1)
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    codes = torch.zeros((8, 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:      # codes without scales
        moe.moe_nvfp4_forward_w4a4(x, lg, bank, act, cfg.k, taps={"x_codes": codes})
    assert ei.value.code == -1


def test_w4a4_code_ties_decided_as_by_division():
    """Activations exactly on E2M1 rounding ties (and block maxima that make the block scale 1
    exactly): the GPU decides such codes by division (ties to even); every x code and scale byte
    equals the oracle's."""
    cfg = moe_inputs.LayerConfig(name="w4a4_ties", E=8, k=2, H=512, I=256, T=16, seed=2)
    buf, bank = device_bank(cfg)
    lg = moe_inputs.make_logits(cfg)
    s = np.float32(2.0 ** -8)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    rng = np.random.default_rng(4)
    x = np.empty((cfg.T, cfg.H), np.float32)
    for t in range(cfg.T):
        for b in range(cfg.H // 16):
            blk = rng.choice(np.concatenate([ties, -ties, ties * 0.5, np.float32([0.5, 1.0, 3.0])]), 16)
            blk[rng.integers(16)] = 6.0 * (1 if rng.random() < 0.5 else -1)   # block maximum 6 s
            x[t, 16 * b:16 * b + 16] = blk * s
    xb = moe_inputs.gen.to_bf16_bits(x)
    assert np.array_equal(oracle.bf16_bits_to_f64(xb), x.astype(np.float64))   # exact in BF16
    act = np.tile(np.array([[s, np.float32(4.0 / 2688)]], np.float32), (cfg.E, 1))
    out, taps = _run(cfg, bank, xb, lg, act)
    _check_slots(cfg, xb, lg, act, taps, range(cfg.T * cfg.k))
