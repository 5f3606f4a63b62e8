import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running")


def load_golden(name: str) -> dict:
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split()[:2]
            vals[key] = int(val)
    return vals


# Output tolerance of the layer against the FP64 oracle.  The layer's output is BF16, so every
# element carries up to half a BF16 spacing of rounding even when computed exactly; the bound
# is 2e-2 * RMS(oracle) on top of that:  |gpu - ref| <= 2e-2 * RMS(ref) + ulp_bf16(ref) / 2 for
# every element, and mean relative error sum|gpu - ref| / sum|ref| <= 3e-3.
MAX_ERR_OVER_RMS = 2e-2
MEAN_REL_ERR = 3e-3


def bf16_half_ulp(ref: np.ndarray) -> np.ndarray:
    """Half the BF16 spacing at |ref| (the rounding error bound of a correctly rounded BF16)."""
    a = np.abs(np.asarray(ref, dtype=np.float64))
    _, e = np.frexp(np.where(a > 0, a, 1.0))          # a = m * 2^e, 0.5 <= m < 1
    return np.ldexp(1.0, np.maximum(e.astype(np.int64) - 9, -134))


def layer_errors(got: np.ndarray, ref: np.ndarray):
    """(max over elements of |err| / allowance, mean relative error, max |err| / RMS)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    allow = MAX_ERR_OVER_RMS * rms + bf16_half_ulp(ref)
    return float((err / allow).max()), float(err.sum() / np.abs(ref).sum()), float(err.max()) / rms


def assert_layer_close(got, ref, what=""):
    a, b, raw = layer_errors(got, ref)
    ok = a <= 1.0 and b <= MEAN_REL_ERR
    dump = os.environ.get("MOE_TEST_DUMP")
    if dump and not ok:
        os.makedirs(dump, exist_ok=True)
        tag = "".join(ch if ch.isalnum() else "_" for ch in what)
        np.savez_compressed(os.path.join(dump, f"fail_{tag}.npz"), got=np.asarray(got), ref=np.asarray(ref))
    assert ok, (f"{what}: max |err| / (2e-2 RMS + ulp/2) = {a:.3f} (<= 1), mean rel = {b:.3e} (<= {MEAN_REL_ERR}),"
                f" max|err|/RMS = {raw:.3e}")
    return a, b


@pytest.fixture(scope="session")
def golden():
    return load_golden
