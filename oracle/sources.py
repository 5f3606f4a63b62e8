"""Expert weights for the oracle, regenerated on the host (test infrastructure only).

A record is rebuilt byte for byte by the seeded generator in ``moe_inputs`` and decoded by
this package's read_record; nothing is read back from a device.
"""
from __future__ import annotations

import moe_inputs

from .nvfp4 import read_record


class GeneratedRecords:
    """Callable e -> (Wg, Wu, Wd) in FP64 for the records of (seed, layer); picklable."""

    def __init__(self, seed: int, layer: int, E: int, H: int, I: int, global_mode: int = 0,
                 scale_kind: str = "config"):
        self.seed, self.layer, self.global_mode, self.scale_kind = seed, layer, global_mode, scale_kind
        self.lay = moe_inputs.record_layout(E, H, I)

    def __call__(self, e: int):
        rec = moe_inputs.record_bytes(self.seed, self.layer, int(e), self.lay, self.global_mode, self.scale_kind)
        L = self.lay
        return read_record(rec, L.H, L.I, L.codes_off, L.scales_off, L.global_off, self.global_mode)
