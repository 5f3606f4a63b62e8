"""The whole layer on the GPU against the FP64 oracle, within the stated tolerance:
max |err| <= 2e-2 * RMS(oracle) and sum|err| / sum|oracle| <= 3e-3.  The large configs are
checked on the seeded 512-token sample; routing is checked in full by test_gpu_route."""
import numpy as np
import pytest

import moe_inputs
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of, device_bank, pool_map

pytestmark = pytest.mark.gpu

PATHS = ["auto", "decode", "prefill"]
_ORACLE_CACHE = {}


def _run(cfg, bank, xb, lg, path="auto", x_next=False):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    x = bf16_tensor(xb)
    logits = torch.from_numpy(lg).cuda()
    xn = torch.empty_like(x) if x_next else None
    p = {"auto": moe.PATH_AUTO, "decode": moe.PATH_DECODE, "prefill": moe.PATH_PREFILL}[path]
    out = moe.moe_nvfp4_forward_ex(x, logits, bank, cfg.k, x_next=xn, path=p)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    return bits_of(out), (bits_of(xn) if x_next else None)


def _prefill_shape_ok(H, I):
    return H % 256 == 0 and I % 256 == 0


def _expect_unsupported(cfg, bank, xb, lg, path):
    """True (after checking the error) when the path cannot take this shape."""
    import nvfp4_weight_only_top_b200 as moe
    if path != "prefill" or _prefill_shape_ok(cfg.H, cfg.I):
        return False
    with pytest.raises(moe.MoeError) as ei:
        _run(cfg, bank, xb, lg, path)
    assert ei.value.code == -2 and "prefill" in str(ei.value)
    return True


def _oracle(cfg, xb, lg, layer=0, tokens=None, global_mode=0, seed=None):
    src = oracle.GeneratedRecords(cfg.seed if seed is None else seed, layer, cfg.E, cfg.H, cfg.I, global_mode)
    return oracle.layer_forward(xb, lg, cfg.k, src, tokens=tokens, map_fn=pool_map)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", ["tiny", "decode_t1", "decode_t64_zipf", "prefill_t8192"])
def test_layer_matches_oracle(name, path):
    cfg = moe_inputs.CONFIGS[name]
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    if _expect_unsupported(cfg, bank, xb, lg, path):
        return
    out, _ = _run(cfg, bank, xb, lg, path)
    tokens = moe_inputs.sample_tokens(cfg.T, 512, cfg.seed)
    if name not in _ORACLE_CACHE:
        _ORACLE_CACHE[name] = _oracle(cfg, xb, lg, tokens=tokens)["out"]
    assert_layer_close(oracle.bf16_bits_to_f64(out[tokens]), _ORACLE_CACHE[name], f"{name}/{path}")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 2, 3, 8, 9, 13, 64, 65, 100])
def test_tiny_ragged_T(T, path):
    """The tiny layer (I = 256 on the tensor-core path, whose K-stages need I % 256 == 0)."""
    base = moe_inputs.CONFIGS["tiny"]
    I = 256 if path == "prefill" else base.I
    cfg = moe_inputs.LayerConfig("tiny_T", base.E, base.k, base.H, I, T, 1, "distinct", seed=T)
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    out, _ = _run(cfg, bank, xb, lg, path)
    assert_layer_close(oracle.bf16_bits_to_f64(out), _oracle(cfg, xb, lg)["out"], f"T={T}/{path}")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("E,k,H,I,T", [(16, 1, 256, 128, 5), (16, 16, 256, 128, 6), (64, 4, 384, 256, 40),
                                       (8, 2, 128, 128, 3), (32, 8, 1024, 512, 20), (16, 4, 512, 256, 37),
                                       (8, 8, 256, 768, 50), (4, 3, 1280, 256, 7)])
def test_shapes(E, k, H, I, T, path):
    cfg = moe_inputs.LayerConfig("shape", E, k, H, I, T, 1, "normal", seed=E + H)
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    if _expect_unsupported(cfg, bank, xb, lg, path):
        return
    out, _ = _run(cfg, bank, xb, lg, path)
    assert_layer_close(oracle.bf16_bits_to_f64(out), _oracle(cfg, xb, lg)["out"], f"{E},{k},{H},{I},{T}/{path}")


@pytest.mark.parametrize("E,k,H,I,T,dist", [
    (8, 2, 256, 256, 1100, "normal"),      # about 275 rows per expert: groups of 256 plus a ragged group
    (4, 4, 512, 256, 600, "normal"),       # every expert takes 600 rows: 256 + 256 + 88
    (16, 2, 768, 512, 300, "zipf"),        # skewed counts, K = 768 / 512: many stages, 3-4 M-tile pairs
    (2, 1, 256, 256, 520, "normal")])      # two experts, groups of 1..256 rows
def test_prefill_groups_beyond_one_tile(E, k, H, I, T, dist):
    cfg = moe_inputs.LayerConfig("prefill_groups", E, k, H, I, T, 1, dist, seed=T + H)
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    ref = _oracle(cfg, xb, lg)["out"]
    for path in ("prefill", "decode"):
        out, _ = _run(cfg, bank, xb, lg, path)
        assert_layer_close(oracle.bf16_bits_to_f64(out), ref, f"{E},{k},{H},{I},{T}/{path}")


@pytest.mark.parametrize("path", PATHS)
def test_global_mode_1(path):
    base = moe_inputs.CONFIGS["tiny"]
    cfg = moe_inputs.LayerConfig("tiny_mode1", base.E, base.k, base.H, 256, base.T, 1, base.logits)
    buf, bank = device_bank(cfg, global_mode=1)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    out, _ = _run(cfg, bank, xb, lg, path)
    assert_layer_close(oracle.bf16_bits_to_f64(out), _oracle(cfg, xb, lg, global_mode=1)["out"], f"mode1/{path}")


def test_T0_enqueues_nothing():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["tiny"]
    buf, bank = device_bank(cfg)
    x = torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((0, cfg.E), dtype=torch.float32, device="cuda")
    moe.moe_nvfp4_forward(x, lg, bank, cfg.k)
    assert moe.moe_nvfp4_last_launch_count() == 0


def test_deterministic_and_workspace_paths_agree():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["decode_t64_zipf"]
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()
    a = moe.moe_nvfp4_forward(x, lg, bank, cfg.k)
    b = moe.moe_nvfp4_forward(x, lg, bank, cfg.k)
    nb = moe.moe_nvfp4_workspace_bytes(cfg.T, cfg.E, cfg.k, cfg.H, cfg.I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    c = moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_forward_host_matches_device_call():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["decode_t1"]
    buf, bank = device_bank(cfg)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    dev = moe.moe_nvfp4_forward(bf16_tensor(xb), torch.from_numpy(lg).cuda(), bank, cfg.k)
    host = moe.moe_nvfp4_forward_host(xb, lg, bank, cfg.k)
    assert np.array_equal(bits_of(dev), host)


def test_forward_host_repeated_calls_replay_correctly():
    """Small host calls replay a captured graph after their first (eager) call: repeated calls
    with new inputs, alternating sizes and banks, pinned and pageable buffers, and a growth of
    the internal workspace in between all equal the device call bit for bit."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfgs = [moe_inputs.LayerConfig("host_a", 16, 4, 1024, 512, 1, seed=3),
            moe_inputs.LayerConfig("host_b", 16, 4, 1024, 512, 3, seed=4),
            moe_inputs.LayerConfig("host_c", 32, 8, 512, 256, 2, seed=5)]
    banks = [device_bank(c) for c in cfgs]
    for it in range(4):
        for ci, cfg in enumerate(cfgs):
            xb = moe_inputs.make_x(cfg, seed=100 + it)
            lg = moe_inputs.make_logits(cfg, seed=200 + it)
            if it % 2:
                xh = torch.from_numpy(xb.view(np.int16)).pin_memory().numpy().view(np.uint16)
                lh = torch.from_numpy(lg).pin_memory().numpy()
            else:
                xh, lh = xb, lg
            dev = moe.moe_nvfp4_forward(bf16_tensor(xb), torch.from_numpy(lg).cuda(), banks[ci][1], cfg.k)
            host = moe.moe_nvfp4_forward_host(xh, lh, banks[ci][1], cfg.k)
            assert np.array_equal(bits_of(dev), host), (it, cfg.name)
        if it == 1:     # grow the internal workspace (a large call), so cached graphs must be rebuilt
            big = moe_inputs.LayerConfig("host_big", 16, 4, 1024, 512, 2048, seed=6)
            bb = device_bank(big)
            moe.moe_nvfp4_forward(bf16_tensor(moe_inputs.make_x(big)), torch.from_numpy(moe_inputs.make_logits(big)).cuda(),
                                  bb[1], big.k)
            torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0


def test_workspace_too_small_is_rejected():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["tiny"]
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, workspace=ws)
    assert ei.value.code == -4


def test_verify24_stack_teacher_forced():
    """24 stacked layers with the residual add: every layer's residual is bit-exact against the
    oracle's rounding of (x + out), and sampled layers match the oracle teacher-forced."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["verify24_t16"]
    lay = cfg.layout
    banks, bufs = [], []
    for l in range(cfg.layers):
        b, bk = device_bank(cfg, layer=l)
        bufs.append(b)
        banks.append(bk)
    xs = [bf16_tensor(moe_inputs.make_x(cfg))]
    outs = []
    for l in range(cfg.layers):
        lg = torch.from_numpy(moe_inputs.make_logits(cfg, layer=l)).cuda()
        xn = torch.empty_like(xs[-1])
        outs.append(moe.moe_nvfp4_forward_ex(xs[-1], lg, banks[l], cfg.k, x_next=xn))
        xs.append(xn)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    xb = [bits_of(t) for t in xs]
    ob = [bits_of(t) for t in outs]
    for l in range(cfg.layers):
        assert np.array_equal(xb[l + 1], oracle.residual_add(xb[l], ob[l])), f"residual layer {l}"
    for l in (0, 11, 23):
        ref = _oracle(cfg, xb[l], moe_inputs.make_logits(cfg, layer=l), layer=l)
        assert_layer_close(oracle.bf16_bits_to_f64(ob[l]), ref["out"], f"layer {l}")


def test_prefill_bitwise_repeatable():
    """The tensor-core path has a fixed summation order: repeated calls give identical bits.  A
    hand-off race between its producer, TMA and MMA roles shows up here as a changed column."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.CONFIGS["prefill_t8192"]
    buf, bank = device_bank(cfg)
    x = bf16_tensor(moe_inputs.make_x(cfg))
    lg = torch.from_numpy(moe_inputs.make_logits(cfg)).cuda()
    first = moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, path=moe.PATH_PREFILL).view(torch.int16).clone()
    for _ in range(6):
        again = moe.moe_nvfp4_forward_ex(x, lg, bank, cfg.k, path=moe.PATH_PREFILL).view(torch.int16)
        torch.cuda.synchronize()
        assert torch.equal(first, again)
    assert moe.moe_nvfp4_device_status() == 0


@pytest.mark.parametrize("E,k,H,I,mode", [(32, 8, 1024, 512, 0), (64, 4, 2048, 1024, 1), (16, 1, 4096, 1536, 0),
                                          (256, 8, 5120, 2560, 1), (8, 8, 1024, 512, 0)])
def test_single_token_fused_kernel(E, k, H, I, mode):
    """T = 1 runs route, gate/up, down and combine in one persistent kernel (one launch); its
    output matches the oracle and its residual is bit-exact."""
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.LayerConfig("single", E, k, H, I, 1, 1, "normal", seed=E + k + H)
    buf, bank = device_bank(cfg, global_mode=mode)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    for path in ("auto", "decode"):
        out, xn = _run(cfg, bank, xb, lg, path, x_next=True)
        assert moe.moe_nvfp4_last_launch_count() == 1
        ref = _oracle(cfg, xb, lg, global_mode=mode)
        assert_layer_close(oracle.bf16_bits_to_f64(out), ref["out"], f"T=1 {E},{k},{H},{I}/{path}")
        assert np.array_equal(xn, oracle.residual_add(xb, out))


@pytest.mark.parametrize("E,k,H,I,T,mode", [(16, 4, 1024, 512, 2, 0), (8, 8, 1024, 512, 3, 1), (64, 8, 2048, 1024, 7, 0),
                                            (32, 8, 1024, 512, 11, 0), (256, 8, 5120, 2560, 11, 0),
                                            (4, 1, 4096, 1536, 11, 1), (32, 8, 1024, 512, 16, 0),
                                            (256, 8, 5120, 2560, 16, 0), (4, 1, 4096, 1536, 16, 1)])
def test_few_tokens_fused_kernel(E, k, H, I, T, mode):
    """2 <= T <= 11 (T k <= the SM count): the router kernel, then one persistent kernel over
    one slot per routed row; slots of one expert repeat its rows (E small forces it).  From 12
    tokens on the grouped kernels take over (router, gate/up, down, combine)."""
    import nvfp4_weight_only_top_b200 as moe
    cfg = moe_inputs.LayerConfig("few", E, k, H, I, T, 1, "normal", seed=E + T + H)
    buf, bank = device_bank(cfg, global_mode=mode)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    ref = _oracle(cfg, xb, lg, global_mode=mode)
    for path in ("auto", "decode"):
        out, xn = _run(cfg, bank, xb, lg, path, x_next=True)
        assert moe.moe_nvfp4_last_launch_count() == (2 if T < 12 else 4)
        assert_layer_close(oracle.bf16_bits_to_f64(out), ref["out"], f"T={T} {E},{k},{H},{I}/{path}")
        assert np.array_equal(xn, oracle.residual_add(xb, out))


def test_prefill_pair_kernel_matches_oracle():
    """The CTA-pair prefill kernel (tcgen05 cta_group::2, selected by MOE_NVFP4_PREFILL=pair when
    the library loads) on full and partial groups, in a fresh process, against the oracle."""
    import os
    import subprocess
    import sys
    code = (
        "import numpy as np, torch, moe_inputs, oracle\n"
        "import nvfp4_weight_only_top_b200 as moe\n"
        "from gpu_helpers import device_bank, bf16_tensor, bits_of\n"
        "from conftest import assert_layer_close\n"
        "for (E, k, H, I, T) in [(16, 8, 512, 256, 700), (8, 2, 1024, 512, 300)]:\n"
        "    cfg = moe_inputs.LayerConfig('pair', E, k, H, I, T, 1, 'normal', seed=T)\n"
        "    buf, bank = device_bank(cfg)\n"
        "    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)\n"
        "    out = moe.moe_nvfp4_forward_ex(bf16_tensor(xb), torch.from_numpy(lg).cuda(), bank, k, path=moe.PATH_PREFILL)\n"
        "    torch.cuda.synchronize()\n"
        "    assert moe.moe_nvfp4_device_status() == 0\n"
        "    ref = oracle.layer_forward(xb, lg, k, oracle.GeneratedRecords(cfg.seed, 0, E, H, I))\n"
        "    assert_layer_close(oracle.bf16_bits_to_f64(bits_of(out)), ref['out'], f'pair {E} {k} {H} {I} {T}')\n"
        "print('pair ok')\n")
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MOE_NVFP4_PREFILL="pair",
               PYTHONPATH=os.pathsep.join([here, os.path.dirname(here), os.environ.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "pair ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
