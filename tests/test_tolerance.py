"""Pins of the output tolerance used by the GPU parity tests (CPU only)."""
import ml_dtypes
import numpy as np

from conftest import bf16_half_ulp, layer_errors


def test_half_ulp_matches_bf16_spacing():
    for x in [0.5, 0.75, 0.99609375, 1.0, 3.0, 2.0 ** -10, -0.625, 2.0 ** -126, 2.0 ** 100]:
        b = np.array([abs(x)], dtype=np.float32).astype(ml_dtypes.bfloat16)
        mag = float(b.astype(np.float64)[0])
        nxt = float((b.view(np.uint16) + np.uint16(1)).view(ml_dtypes.bfloat16).astype(np.float64)[0])
        assert bf16_half_ulp(np.array([x]))[0] == (nxt - mag) / 2, x


def test_correct_bf16_rounding_always_passes():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(100000) * np.exp(rng.standard_normal(100000))   # heavy tails
    got = ref.astype(ml_dtypes.bfloat16).astype(np.float64)
    a, b, raw = layer_errors(got, ref)
    assert a <= 1.0 and b <= 3e-3
    # the plain 2e-2 * RMS bound alone would reject correctly rounded outputs here
    assert raw > 2e-2


def test_the_worst_case_seen_on_the_batched_decode_config():
    # exact 0.5019418997; the GPU's f32 sum rounded up to 0.50390625 (one BF16 step above the
    # correctly rounded 0.5); RMS of the whole output 0.0803817
    ref = np.array([0.5019418997378996] + [0.0803817] * 99)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    got = ref.copy()
    got[0] = 0.50390625
    a, _, raw = layer_errors(got, ref)
    assert a <= 1.0 and raw / rms * rms > 0


def test_real_errors_fail():
    rng = np.random.default_rng(1)
    ref = rng.standard_normal(10000)
    got = ref.copy()
    got[17] += 0.05 * np.sqrt(np.mean(ref ** 2))          # 5% of RMS on one element
    assert layer_errors(got, ref)[0] > 1.0
    got = ref * (1 + 4e-3)                                 # 0.4% everywhere
    assert layer_errors(got, ref)[1] > 3e-3
