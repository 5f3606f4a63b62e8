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


# Output tolerance of the layer against the FP64 oracle: max |err| <= 2e-2 * RMS(oracle)
# and mean relative error sum|err| / sum|ref| <= 3e-3.
MAX_ERR_OVER_RMS = 2e-2
MEAN_REL_ERR = 3e-3


def layer_errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(err.max()) / rms, float(err.sum() / np.abs(ref).sum())


def assert_layer_close(got, ref, what=""):
    a, b = layer_errors(got, ref)
    assert a <= MAX_ERR_OVER_RMS and b <= MEAN_REL_ERR, \
        f"{what}: max|err|/rms={a:.3e} (<= {MAX_ERR_OVER_RMS}), mean rel={b:.3e} (<= {MEAN_REL_ERR})"
    return a, b


@pytest.fixture(scope="session")
def golden():
    return load_golden
