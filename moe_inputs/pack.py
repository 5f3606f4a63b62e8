"""Writes a synthetic streaming pack in the layout of the page "Beam 1.0 501B-A23B, streaming pack,
NVFP4 experts / MLX 8-bit residents" (section "What this pack holds"): experts.bin holds one record
per (layer, expert), every record starting at a multiple of 4 KiB, and expert-manifest.json names
the format and layout, the source pin, the 9 parts of a record, and the offset, length and sha256
of each record, plus the list of projections whose global scale is inexact.

The record bytes are the seeded generator's (record_bytes, global mode 1: the stored f32 is the
pack's g, whose multiplier is f32(g / 2688)).  The page prints the manifest's fields but not its
JSON schema; the schema written here is this library's reading of it:

  {"format": "mlx-stream-nvfp4-expert-bank-v1", "layout": "nvfp4-gud-9part",
   "source": {"repo": ..., "revision": ...},
   "layers": L, "experts": E, "hidden": H, "intermediate": I,
   "record_bytes": ..., "record_stride": ...,
   "parts": [{"name": "gate.codes", "offset": ..., "length": ...}, ... 9 parts],
   "records": [{"layer": l, "expert": e, "offset": ..., "length": ..., "sha256": "<hex>"}, ...],
   "global_scale_inexact": [{"layer": l, "expert": e, "projection": "gate"}, ...]}

Records are stored layer-major (record index = layer * E + expert).  Only random bytes are drawn
here; nothing of the layer's arithmetic is computed.
"""
from __future__ import annotations

import hashlib
import json
import os

import numpy as np

from .gen import record_bytes, record_layout

FORMAT = "mlx-stream-nvfp4-expert-bank-v1"
LAYOUT = "nvfp4-gud-9part"
PART_NAMES = ("gate.codes", "up.codes", "down.codes", "gate.scales", "up.scales", "down.scales",
              "gate.global", "up.global", "down.global")


def write_pack(directory: str, layers: int, E: int, H: int, I: int, seed: int = 0,
               inexact=(), corrupt=()) -> dict:
    """Writes experts.bin and expert-manifest.json into directory; returns the manifest.

    inexact: (layer, expert, projection name) entries listed as global_scale_inexact.
    corrupt: (layer, expert) records whose bytes are altered after their sha256 was taken (for
    tests of the loader's integrity check).
    """
    os.makedirs(directory, exist_ok=True)
    lay = record_layout(E, H, I)
    sizes = [H * I // 2] * 3 + [H * I // 16] * 3 + [4] * 3
    offs = list(lay.codes_off) + list(lay.scales_off) + list(lay.global_off)
    parts = [{"name": n, "offset": int(o), "length": int(s)} for n, o, s in zip(PART_NAMES, offs, sizes)]
    records = []
    bad = {tuple(c) for c in corrupt}
    with open(os.path.join(directory, "experts.bin"), "wb") as f:
        for layer in range(layers):
            for e in range(E):
                rec = record_bytes(seed, layer, e, lay, global_mode=1)
                off = (layer * E + e) * lay.record_stride
                records.append({"layer": layer, "expert": e, "offset": off, "length": lay.record_bytes,
                                "sha256": hashlib.sha256(rec.tobytes()).hexdigest()})
                if (layer, e) in bad:
                    rec = rec.copy()
                    rec[len(rec) // 3] ^= 0x40
                f.seek(off)
                f.write(rec.tobytes())
        f.truncate(layers * E * lay.record_stride)
    manifest = {"format": FORMAT, "layout": LAYOUT,
                "source": {"repo": "synthetic", "revision": f"seed-{seed}"},
                "layers": layers, "experts": E, "hidden": H, "intermediate": I,
                "record_bytes": lay.record_bytes, "record_stride": lay.record_stride,
                "parts": parts, "records": records,
                "global_scale_inexact": [{"layer": int(l), "expert": int(e), "projection": p}
                                         for (l, e, p) in inexact]}
    with open(os.path.join(directory, "expert-manifest.json"), "w") as f:
        json.dump(manifest, f, indent=1)
    return manifest


def pack_record(directory: str, layer: int, expert: int) -> np.ndarray:
    """The bytes of one record as stored in experts.bin (for tests)."""
    with open(os.path.join(directory, "expert-manifest.json")) as f:
        m = json.load(f)
    r = m["records"][layer * m["experts"] + expert]
    with open(os.path.join(directory, "experts.bin"), "rb") as f:
        f.seek(r["offset"])
        return np.frombuffer(f.read(r["length"]), dtype=np.uint8)
