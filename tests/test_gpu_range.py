"""The decode kernels over the whole range of the layer's inputs, against the FP64 oracle.

The CUDA-core and mma.sync decode kernels multiply the weights with the activations in f16,
whose range (6e-8 .. 65504) is far narrower than BF16's; they first scale each activation
vector (a token's x, a routed row's mid values h) by an exact power of two taken from its
largest magnitude.  These tests feed:
  * tokens whose scale ranges from 2^-30 to 2^17 in one call, and heavy-tailed rows;
  * layers whose mid values h reach far beyond f16 (above 1e5);
  * E4M3 block scales over every non-NaN encoding (zero, subnormals, negative, up to 448);
on every path (the single-token kernel at T = 1, the few-token kernel, the batched kernels and
the tensor-core path), and compare each token with the oracle on its own (the tolerance is
relative to that token's RMS, so a small token is not hidden behind a large one).

The page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section
"What this pack holds", keeps the activations in BF16: the layer must hold for any BF16 input
whose result is finite.
"""
import numpy as np
import pytest

import moe_inputs
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of, pool_map

pytestmark = pytest.mark.gpu

EXPS = [-30, -12, 0, 9, 17, 4, -3]           # per-token scale exponents (max |x| up to ~2^19)


def _bank_from_host(cfg, scale_kind):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    lay = cfg.layout
    host = moe_inputs.gen.bank_host(cfg.seed, 0, lay, 0, scale_kind)
    buf = torch.from_numpy(host).cuda()
    bank = moe.make_bank(buf.data_ptr(), lay.E, lay.H, lay.I, lay.record_stride, lay.codes_off, lay.scales_off,
                         lay.global_off, 0)
    return buf, bank


def _run(cfg, bank, xb, lg, path):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    p = {"auto": moe.PATH_AUTO, "decode": moe.PATH_DECODE, "prefill": moe.PATH_PREFILL}[path]
    x = bf16_tensor(xb)
    xn = torch.empty_like(x)
    out = moe.moe_nvfp4_forward_ex(x, torch.from_numpy(lg).cuda(), bank, cfg.k, x_next=xn, path=p)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_device_status() == 0
    return bits_of(out), bits_of(xn)


def _check_per_token(cfg, xb, lg, out, xn, scale_kind, what):
    src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I, 0, scale_kind)
    ref = oracle.layer_forward(xb, lg, cfg.k, src, map_fn=pool_map)["out"]
    got = oracle.bf16_bits_to_f64(out)
    assert np.all(np.isfinite(ref))
    for t in range(cfg.T):
        assert_layer_close(got[t], ref[t], f"{what} token {t}")
    assert np.array_equal(xn, oracle.residual_add(xb, out))


@pytest.mark.parametrize("scale_kind", ["config", "all_finite"])
@pytest.mark.parametrize("path", ["auto", "decode", "prefill"])
@pytest.mark.parametrize("T", [1, 5, 24])
def test_wide_activations(T, path, scale_kind):
    """E=16, k=4, H=1024, I=512: T = 1 takes the single-token kernel, T = 5 the few-token
    kernel, T = 24 the batched kernels (all on the decode path); T = 1 runs once per scale."""
    cfg = moe_inputs.LayerConfig("wide", 16, 4, 1024, 512, T, 1, "normal", seed=T + 7)
    buf, bank = _bank_from_host(cfg, scale_kind)
    lg = moe_inputs.make_logits(cfg)
    runs = [[e] for e in EXPS] if T == 1 else [EXPS]
    for exps in runs:
        for heavy in (False, True):
            xb = moe_inputs.make_x_wide(T, cfg.H, exps, seed=1000 + T + exps[0] + 100 * heavy, heavy=heavy)
            out, xn = _run(cfg, bank, xb, lg, path)
            _check_per_token(cfg, xb, lg, out, xn, scale_kind, f"T={T} {path} {scale_kind} exps={exps} heavy={heavy}")


@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_mid_values_far_beyond_f16(path):
    """Tokens of scale 2^12: the oracle's mid values h = silu(Wg x) (Wu x) exceed 1e5 (f16 tops
    out at 65504), so the h prescale of the down projection is exercised."""
    cfg = moe_inputs.LayerConfig("bigh", 16, 4, 1024, 512, 3, 1, "normal", seed=11)
    buf, bank = _bank_from_host(cfg, "config")
    lg = moe_inputs.make_logits(cfg)
    xb = moe_inputs.make_x_wide(cfg.T, cfg.H, [12], seed=5)
    src = oracle.GeneratedRecords(cfg.seed, 0, cfg.E, cfg.H, cfg.I)
    ids, _ = oracle.route(lg, cfg.k)
    Wg, Wu, _ = src(int(ids[0, 0]))
    x0 = oracle.bf16_bits_to_f64(xb[0])
    h = oracle.silu(Wg @ x0) * (Wu @ x0)
    assert np.abs(h).max() > 1e5
    for T in (1, 3):                          # the single-token and the few-token kernels
        sub = moe_inputs.LayerConfig("bigh", 16, 4, 1024, 512, T, 1, "normal", seed=11)
        out, xn = _run(sub, bank, xb[:T], lg[:T], path)
        _check_per_token(sub, xb[:T], lg[:T], out, xn, "config", f"big h T={T} {path}")


def _workspace_routing(T, k, ws):
    import torch
    R = T * k
    raw = ws.cpu().numpy()
    ids = raw[:R * 4].view(np.int32).reshape(T, k)
    off = 256 * -(-R * 4 // 256)
    w = raw[off:off + R * 4].view(np.float32).reshape(T, k)
    return ids, w


def _special_logits(E, rng):
    rows = []
    rows.append(rng.integers(-2, 3, E).astype(np.float32))                    # many exact ties
    r = np.zeros(E, np.float32); r[::3] = -0.0; r[5] = 0.0; rows.append(r)   # -0.0 ties +0.0
    r = np.full(E, -np.inf, np.float32); r[[3, E - 56, E // 3]] = [1.0, 1.0, -5.0]; rows.append(r)
    r = rng.standard_normal(E).astype(np.float32); r[:40] = np.nan; rows.append(r)
    rows.append(np.full(E, np.nan, np.float32))                               # NaN: by index
    r = rng.standard_normal(E).astype(np.float32); r[17] = np.inf; rows.append(r)
    r = np.full(E, 5.0, np.float32); r[::7] = 6.0; rows.append(r)             # 37 at the top
    rows.append((rng.standard_normal(E) * 1e-39).astype(np.float32))          # subnormal logits
    r = rng.standard_normal(E).astype(np.float32); r[E - 56:] = 50.0; rows.append(r)
    return rows


@pytest.mark.parametrize("E", [256, 64])
def test_single_token_router_bit_exact(E):
    """The single-token kernel ranks the experts inside the kernel (its own rank count, not the
    router kernel): its ids must equal the oracle's bit for bit, ties to the lower index, -0.0
    equal to +0.0, NaN below -inf, and its weights must match to f32 rounding; where every
    weight is finite the layer output is checked too."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    k = 8
    cfg = moe_inputs.LayerConfig("route1", E, k, 1024, 512, 1, 1, "normal", seed=E)
    buf, bank = _bank_from_host(cfg, "config")
    xb = moe_inputs.make_x(cfg)
    ws = torch.empty(moe.moe_nvfp4_workspace_bytes(1, E, k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(E)
    for i, row in enumerate(_special_logits(E, rng)):
        lg = row[None, :].copy()
        x = bf16_tensor(xb)
        out = moe.moe_nvfp4_forward_ex(x, torch.from_numpy(lg).cuda(), bank, k, workspace=ws)
        torch.cuda.synchronize()
        assert moe.moe_nvfp4_last_launch_count() == 1          # the fused single-token kernel
        assert moe.moe_nvfp4_device_status() == 0
        ids, w = _workspace_routing(1, k, ws)
        rid, rw = oracle.route(lg, k)
        assert np.array_equal(ids, rid), (i, ids, rid)
        fin = np.isfinite(rw)
        assert np.array_equal(np.isfinite(w), fin), i
        assert np.allclose(w[fin], rw[fin], rtol=2e-6, atol=1e-7), i
        if fin.all():
            src = oracle.GeneratedRecords(cfg.seed, 0, E, cfg.H, cfg.I)
            ref = oracle.layer_forward(xb, lg, k, src, map_fn=pool_map)["out"]
            assert_layer_close(oracle.bf16_bits_to_f64(bits_of(out)), ref, f"router case {i}")
