"""Pins of the oracle's routing, permutation, layer and residual (CPU only).

Each test checks the oracle against something other than itself: library routines
(torch.softmax, torch.nn.functional.silu, torch matmul, ml_dtypes BF16 rounding), closed
forms (k = 2 weights are a logistic function of the logit gap), brute force (full sort,
dense masked sum over all experts), special cases (k = 1, k = E) and invariances
(relabelling experts, power-of-two down scaling).
"""

import ml_dtypes
import numpy as np
import pytest
import torch

import moe_inputs
import oracle


# ---------------------------------------------------------------- routing

def _brute_route(lg, k):
    T, E = lg.shape
    ids = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        def key(e):
            v = float(lg[t, e])
            return (1, 0.0, e) if v != v else (0, -v, e)
        ids[t] = sorted(range(E), key=key)[:k]
    return ids


@pytest.mark.parametrize("E,k", [(16, 2), (256, 8), (64, 1), (32, 32)])
def test_route_matches_full_sort(E, k):
    lg = np.random.default_rng(E + k).standard_normal((40, E)).astype(np.float32)
    ids, w = oracle.route(lg, k)
    assert np.array_equal(ids, _brute_route(lg, k))
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # weights are non-increasing with rank
    assert np.all(np.diff(w, axis=1) <= 0)


def test_route_k1_weight_is_one():
    lg = np.random.default_rng(1).standard_normal((10, 16)).astype(np.float32)
    ids, w = oracle.route(lg, 1)
    assert np.array_equal(ids[:, 0], lg.argmax(axis=1)) and np.all(w == 1.0)


def test_route_k2_closed_form():
    lg = np.random.default_rng(2).standard_normal((50, 16)).astype(np.float32)
    ids, w = oracle.route(lg, 2)
    d = lg[np.arange(50), ids[:, 0]].astype(np.float64) - lg[np.arange(50), ids[:, 1]]
    p = 1.0 / (1.0 + np.exp(-d))                    # logistic of the gap
    assert np.allclose(w[:, 0], p, rtol=1e-14) and np.allclose(w[:, 1], 1 - p, rtol=1e-13)


def test_route_k_equals_E_is_full_softmax():
    lg = np.random.default_rng(3).standard_normal((8, 16)).astype(np.float32)
    ids, w = oracle.route(lg, 16)
    ref = torch.softmax(torch.from_numpy(lg.astype(np.float64)), dim=1).numpy()
    full = np.zeros_like(ref)
    full[np.arange(8)[:, None], ids] = w
    assert np.allclose(full, ref, rtol=1e-14, atol=0)


def test_route_ties_go_to_lower_index():
    E = 16
    lg = np.zeros((4, E), dtype=np.float32)
    lg[1, [3, 9, 12]] = 1.0                   # three equal maxima
    lg[2] = -0.0
    lg[2, [5, 7]] = 0.0                        # -0.0 and +0.0 tie
    lg[3, :] = -np.inf
    lg[3, 10] = 2.0
    ids, w = oracle.route(lg, 4)
    assert ids[0].tolist() == [0, 1, 2, 3]
    assert ids[1].tolist() == [3, 9, 12, 0]
    assert ids[2].tolist() == [0, 1, 2, 3]
    assert ids[3].tolist() == [10, 0, 1, 2]
    assert w[3].tolist() == [1.0, 0.0, 0.0, 0.0]
    assert np.allclose(w[0], 0.25)


def test_route_nan_ranks_below_minus_inf():
    lg = np.array([[np.nan, -np.inf, 1.0, np.nan, 0.5]], dtype=np.float32)
    ids, w = oracle.route(lg, 4)
    assert ids[0].tolist() == [2, 4, 1, 0]
    assert np.all(np.isnan(w))                  # a selected NaN poisons the softmax
    ids, w = oracle.route(lg, 3)
    assert ids[0].tolist() == [2, 4, 1] and not np.any(np.isnan(w))


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (8, 16, 2), (300, 64, 4)])
def test_permute_brute_force(T, E, k):
    lg = np.random.default_rng(T).standard_normal((T, E)).astype(np.float32)
    ids, _ = oracle.route(lg, k)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
    p = 0
    for e in range(E):
        rows = [t * k + j for t in range(T) for j in range(k) if ids[t, j] == e]
        assert counts[e] == len(rows) and offsets[e] == p
        assert perm[p:p + len(rows)].tolist() == rows
        p += len(rows)
    assert np.array_equal(perm[inv], np.arange(T * k))


# ---------------------------------------------------------------- layer

def _small_bank(E, H, I, seed=5, mode=0):
    lay = moe_inputs.record_layout(E, H, I)
    recs = [moe_inputs.record_bytes(seed, 0, e, lay, mode) for e in range(E)]
    weights = [oracle.read_record(r, H, I, lay.codes_off, lay.scales_off, lay.global_off, mode)
               for r in recs]
    return lay, recs, weights


def _x_bits(T, H, seed):
    return moe_inputs.gen.to_bf16_bits(np.random.default_rng(seed).standard_normal((T, H)))


def test_silu_matches_torch():
    g = np.linspace(-30, 30, 2001)
    ref = torch.nn.functional.silu(torch.from_numpy(g)).numpy()
    assert np.allclose(oracle.silu(g), ref, rtol=1e-15, atol=1e-300)


def test_layer_k1_is_dense_swiglu_mlp():
    E, H, I, T = 4, 32, 16, 6
    lay, recs, W = _small_bank(E, H, I)
    xb = _x_bits(T, H, 1)
    lg = np.random.default_rng(2).standard_normal((T, E)).astype(np.float32)
    res = oracle.layer_forward(xb, lg, 1, lambda e: W[e])
    x = torch.from_numpy(xb.view(ml_dtypes.bfloat16).astype(np.float64))
    for t in range(T):
        e = int(np.argmax(lg[t]))
        Wg, Wu, Wd = (torch.from_numpy(m) for m in W[e])
        ref = (torch.nn.functional.silu(x[t] @ Wg.T) * (x[t] @ Wu.T)) @ Wd.T
        assert np.allclose(res["out"][t], ref.numpy(), rtol=1e-12, atol=1e-15)


def test_layer_gate_and_up_are_not_interchangeable():
    E, H, I, T = 2, 32, 16, 3
    lay, recs, W = _small_bank(E, H, I)
    xb = _x_bits(T, H, 3)
    lg = np.array([[1.0, 0.0]] * T, dtype=np.float32)
    a = oracle.layer_forward(xb, lg, 1, lambda e: W[e])["out"]
    b = oracle.layer_forward(xb, lg, 1, lambda e: (W[e][1], W[e][0], W[e][2]))["out"]
    assert not np.allclose(a, b)


def test_layer_equals_dense_masked_brute_force():
    cfg = moe_inputs.CONFIGS["tiny"]
    lay, recs, W = _small_bank(cfg.E, cfg.H, cfg.I, seed=0)
    xb = moe_inputs.make_x(cfg)
    lg = moe_inputs.make_logits(cfg)
    res = oracle.layer_forward(xb, lg, cfg.k, lambda e: W[e])
    x = oracle.bf16_bits_to_f64(xb)
    out = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        order = sorted(range(cfg.E), key=lambda e: (-float(lg[t, e]), e))[:cfg.k]
        sel = np.array([lg[t, e] for e in order], dtype=np.float64)
        ws = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
        for e in range(cfg.E):                  # every expert, masked
            if e not in order:
                continue
            Wg, Wu, Wd = W[e]
            h = np.zeros(cfg.I)
            for i in range(cfg.I):
                g = sum(Wg[i, c] * x[t, c] for c in range(cfg.H))
                u = sum(Wu[i, c] * x[t, c] for c in range(cfg.H))
                h[i] = g / (1 + np.exp(-g)) * u
            y = np.array([sum(Wd[o, i] * h[i] for i in range(cfg.I)) for o in range(cfg.H)])
            out[t] += ws[order.index(e)] * y
    assert np.allclose(res["out"], out, rtol=1e-11, atol=1e-14)


def test_layer_invariant_under_expert_relabelling():
    E, H, I, T, k = 8, 32, 16, 10, 3
    lay, recs, W = _small_bank(E, H, I)
    xb = _x_bits(T, H, 4)
    lg = np.random.default_rng(5).standard_normal((T, E)).astype(np.float32)
    pi = np.random.default_rng(6).permutation(E)        # new label of expert e is pi[e]
    lg2 = np.empty_like(lg)
    lg2[:, pi] = lg
    W2 = [None] * E
    for e in range(E):
        W2[pi[e]] = W[e]
    a = oracle.layer_forward(xb, lg, k, lambda e: W[e])
    b = oracle.layer_forward(xb, lg2, k, lambda e: W2[e])
    assert np.allclose(a["out"], b["out"], rtol=1e-13, atol=1e-16)
    assert np.array_equal(pi[a["ids"]], b["ids"])


def test_down_global_power_of_two_scales_output_exactly():
    E, H, I, T, k = 4, 32, 16, 5, 2
    lay = moe_inputs.record_layout(E, H, I)
    xb = _x_bits(T, H, 8)
    lg = np.random.default_rng(9).standard_normal((T, E)).astype(np.float32)
    recs = [moe_inputs.record_bytes(2, 0, e, lay) for e in range(E)]
    W1 = [oracle.read_record(r, H, I, lay.codes_off, lay.scales_off, lay.global_off) for r in recs]
    recs2 = []
    for r in recs:
        r2 = r.copy()
        g = r2[lay.global_off[2]:lay.global_off[2] + 4].view('<f4')
        g[0] = g[0] * np.float32(4.0)
        recs2.append(r2)
    W2 = [oracle.read_record(r, H, I, lay.codes_off, lay.scales_off, lay.global_off) for r in recs2]
    a = oracle.layer_forward(xb, lg, k, lambda e: W1[e])["out"]
    b = oracle.layer_forward(xb, lg, k, lambda e: W2[e])["out"]
    assert np.array_equal(b, 4.0 * a)


def test_global_mode_1_matches_mode_0_when_multipliers_agree():
    E, H, I, T, k = 4, 32, 16, 4, 2
    lay = moe_inputs.record_layout(E, H, I)
    xb = _x_bits(T, H, 10)
    lg = np.random.default_rng(11).standard_normal((T, E)).astype(np.float32)
    W0, W1 = [], []
    for e in range(E):
        r0 = moe_inputs.record_bytes(4, 0, e, lay, 0)
        r1 = r0.copy()
        for p in range(3):
            g = r1[lay.global_off[p]:lay.global_off[p] + 4].view('<f4')
            g[0] = np.float32(2688.0) * np.float32(0.25)          # f32(g / 2688) = 0.25 exactly
            g0 = r0[lay.global_off[p]:lay.global_off[p] + 4].view('<f4')
            g0[0] = np.float32(0.25)
        W0.append(oracle.read_record(r0, H, I, lay.codes_off, lay.scales_off, lay.global_off, 0))
        W1.append(oracle.read_record(r1, H, I, lay.codes_off, lay.scales_off, lay.global_off, 1))
    a = oracle.layer_forward(xb, lg, k, lambda e: W0[e])["out"]
    b = oracle.layer_forward(xb, lg, k, lambda e: W1[e])["out"]
    assert np.array_equal(a, b)


def test_token_subset_matches_full():
    cfg = moe_inputs.CONFIGS["tiny"]
    lay, recs, W = _small_bank(cfg.E, cfg.H, cfg.I, seed=0)
    xb, lg = moe_inputs.make_x(cfg), moe_inputs.make_logits(cfg)
    full = oracle.layer_forward(xb, lg, cfg.k, lambda e: W[e])
    sub = oracle.layer_forward(xb, lg, cfg.k, lambda e: W[e], tokens=[1, 5, 6])
    assert np.allclose(sub["out"], full["out"][[1, 5, 6]], rtol=1e-12, atol=1e-16)


# ---------------------------------------------------------------- BF16 rounding / residual

def test_round_to_bf16_matches_ml_dtypes_on_f32_values():
    rng = np.random.default_rng(12)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000),
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 3.4e38, 1e-40, -1e-44, 2 ** -133, 2 ** -134,
                  1.00390625, 1.01171875]),            # ties: 1 + 2^-8 and 1 + 3 * 2^-8
    ]).astype(np.float32)
    ref = v.astype(ml_dtypes.bfloat16).view(np.uint16)
    got = oracle.round_to_bf16_bits(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_residual_is_exact_sum_rounded_once():
    rng = np.random.default_rng(13)
    a = moe_inputs.gen.to_bf16_bits(rng.standard_normal(50000) * 10.0 ** rng.integers(-6, 6, 50000))
    b = moe_inputs.gen.to_bf16_bits(rng.standard_normal(50000) * 10.0 ** rng.integers(-6, 6, 50000))
    got = oracle.residual_add(a, b)
    # brute force with exact rationals for a sample
    from fractions import Fraction
    av = oracle.bf16_bits_to_f64(a)
    bv = oracle.bf16_bits_to_f64(b)
    for i in range(0, 50000, 997):
        s = Fraction(av[i]) + Fraction(bv[i])
        r = oracle.bf16_bits_to_f64(got[i:i + 1])[0]
        # nothing representable is closer; on a tie the even pattern wins
        lo = oracle.bf16_bits_to_f64(np.array([(int(got[i]) - 1) & 0xFFFF], dtype=np.uint16))[0]
        hi = oracle.bf16_bits_to_f64(np.array([(int(got[i]) + 1) & 0xFFFF], dtype=np.uint16))[0]
        d = abs(Fraction(r) - s)
        for nb in (lo, hi):
            if np.isfinite(nb):
                dn = abs(Fraction(nb) - s)
                assert d < dn or (d == dn and int(got[i]) % 2 == 0)
