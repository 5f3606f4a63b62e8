"""The device bank writer produces the same bytes as the host generator."""
import numpy as np
import pytest

import moe_inputs
from moe_inputs import device as mdev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("E,H,I,mode", [(16, 256, 128, 0), (4, 5120, 2560, 0), (3, 384, 256, 1)])
def test_device_bank_equals_host_records(E, H, I, mode):
    lay = moe_inputs.record_layout(E, H, I)
    buf = mdev.bank_tensor(lay, 11, 2, mode).cpu().numpy()
    for e in range(E):
        rec = moe_inputs.record_bytes(11, 2, e, lay, mode)
        o = e * lay.record_stride
        assert np.array_equal(buf[o:o + lay.record_bytes], rec), e
