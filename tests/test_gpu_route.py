"""Routing on the GPU against the oracle: ids, counts, offsets, perm and inv bit-exact, softmax
weights to f32 rounding (the kernel computes them in f32, the oracle in FP64)."""
import numpy as np
import pytest

import moe_inputs
import oracle

pytestmark = pytest.mark.gpu


def _route_gpu(lg, k):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    r = moe.moe_nvfp4_route(torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    return {kk: v.cpu().numpy() for kk, v in r.items()}


def _check(lg, k):
    got = _route_gpu(lg, k)
    ids, w = oracle.route(lg, k)
    counts, offsets, perm, inv = oracle.permute(ids, lg.shape[1])
    assert np.array_equal(got["ids"], ids)
    assert np.array_equal(got["counts"], counts)
    assert np.array_equal(got["offsets"], offsets)
    assert np.array_equal(got["perm"], perm)
    assert np.array_equal(got["inv"], inv)
    fin = np.isfinite(w)
    assert np.array_equal(np.isfinite(got["w"]), fin)
    assert np.allclose(got["w"][fin], w[fin], rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("name", list(moe_inputs.CONFIGS))
def test_route_configs(name):
    cfg = moe_inputs.CONFIGS[name]
    for layer in range(min(cfg.layers, 3)):
        _check(moe_inputs.make_logits(cfg, layer=layer), cfg.k)


@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 129, 1000])
@pytest.mark.parametrize("E,k", [(16, 1), (16, 16), (64, 4), (256, 8), (300, 32), (1024, 8)])
def test_route_shapes(T, E, k):
    lg = np.random.default_rng(T * 1000 + E + k).standard_normal((T, E)).astype(np.float32)
    _check(lg, k)


def test_route_ties_and_specials():
    E, k, T = 256, 8, 70
    rng = np.random.default_rng(5)
    lg = rng.integers(-2, 3, (T, E)).astype(np.float32)      # many exact ties
    lg[0] = 0.0
    lg[1] = -0.0
    lg[1, ::3] = 0.0                                           # -0.0 / +0.0 ties
    lg[2] = -np.inf
    lg[2, 200] = 1.0
    lg[3, :10] = np.nan                                        # NaN ranks last
    lg[4] = np.nan
    lg[5, 17] = np.inf
    lg[6] = rng.standard_normal(E).astype(np.float32) * 1e-38  # subnormal-scale values
    _check(lg, k)


def test_route_T0():
    import torch
    import nvfp4_weight_only_top_b200 as moe
    r = moe.moe_nvfp4_route(torch.empty((0, 256), dtype=torch.float32, device="cuda"), 8)
    torch.cuda.synchronize()
    assert int(r["counts"].sum()) == 0 and int(r["offsets"].abs().sum()) == 0
