"""The seeded input generators' stated properties (CPU only), checked with the oracle's router."""
import numpy as np
import pytest

import moe_inputs
import oracle


@pytest.mark.parametrize("E,k,sets,window", [(256, 8, 64, 8), (256, 8, 4, 8), (16, 2, 6, 2), (64, 4, 12, 4)])
def test_rotating_logit_sets_never_repeat_an_expert_within_the_window(E, k, sets, window):
    lg = moe_inputs.disjoint_routing_logits(E, k, sets, window, seed=3)
    assert lg.shape == (sets, 1, E) and lg.dtype == np.float32
    ids = [set(oracle.route(lg[s], k)[0][0].tolist()) for s in range(sets)]
    for s in range(sets):
        assert len(np.unique(lg[s, 0])) == E                 # no ties: the top k is unambiguous
        for d in range(1, min(window, sets)):                # the sets are used in a loop
            assert not ids[s] & ids[(s - d) % sets], (s, d)


def test_zipf_logits_favour_the_popular_experts():
    cfg = moe_inputs.CONFIGS["decode_t64_zipf"]
    lg = moe_inputs.make_logits(cfg, T=2048)
    ids, _ = oracle.route(lg, cfg.k)
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    top = np.sort(counts)[::-1]
    # p(e) proportional to 1 / (1 + rank): the most popular expert is picked by most tokens,
    # the tail by few; a uniform router would give every expert about T k / E = 64 rows.
    assert top[0] > 1000 and top[-1] < 64 and (counts > 0).sum() > 200


def test_all_finite_scale_bytes_cover_every_non_nan_e4m3_encoding():
    lay = moe_inputs.record_layout(2, 512, 256)
    rec = moe_inputs.record_bytes(3, 0, 1, lay, 0, "all_finite")
    sc = rec[lay.scales_off[0]:lay.global_off[0]]
    assert set(np.unique(sc).tolist()) == set(range(256)) - {0x7F, 0xFF}
    same = moe_inputs.record_bytes(3, 0, 1, lay, 0, "config")
    assert np.array_equal(rec[:lay.scales_off[0]], same[:lay.scales_off[0]])     # codes do not change


def test_wide_activations_follow_their_per_token_exponents():
    exps = [-30, -8, 0, 9, 17]
    x = moe_inputs.make_x_wide(10, 1024, exps, seed=1)
    v = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(10):
        rms = np.sqrt(np.mean(v[t] ** 2))
        assert 0.8 < rms / 2.0 ** exps[t % 5] < 1.25
