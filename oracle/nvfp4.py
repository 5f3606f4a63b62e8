"""NVFP4 expert-weight decoding, FP64 (oracle; test infrastructure only).

Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section
"What this pack holds": each projection of a record is E2M1 codes in U32 words, one E4M3
block scale for each 16 inputs, and one F32 global scale; a weight is
e2m1(code) x e4m3(block scale) x global.  The same section says MLX takes the block's
scale as e4m3(block scale) x (g / 2688) in f32, with g the stored f32 value; 2688 is the
product of the largest E2M1 magnitude (6) and the largest finite E4M3 magnitude (448).

Readings where the page is silent (each listed in the design notes):
  * E2M1 is the OCP Microscaling FP4 format: sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0; exponent 0 is subnormal (0 or 0.5); no inf or NaN.
  * E4M3 is the OCP "FN" variant: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits
    2..0; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no inf.
  * Inside a projection the weights are row-major [out, in]; element 8w + n of a row is the
    4-bit field at bits 4n .. 4n+3 of little-endian word w of that row (low nibble first).
  * Block scales are row-major [out, in/16]: scale (o, b) covers inputs 16b .. 16b+15.
  * global_mode 0: the stored f32 is the multiplier itself; global_mode 1: the stored f32
    is g and the multiplier is f32(g / 2688), computed in f32 as the page says MLX does.
"""
from __future__ import annotations

import math

import numpy as np


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code from its bit fields."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        mag = 0.5 * m                      # subnormal: 2^(1-bias) * (m / 2), bias 1
    else:
        mag = 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return -mag if s else mag


def e4m3_value(byte: int) -> float:
    """Value of an E4M3 (FN) byte from its bit fields."""
    s = (byte >> 7) & 1
    e = (byte >> 3) & 15
    m = byte & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        mag = 2.0 ** -6 * (m / 8.0)        # subnormal: 2^(1-bias) * (m / 8), bias 7
    else:
        mag = 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return -mag if s else mag


E2M1_VALUES = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_VALUES = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)


def projection_bytes(out_features: int, in_features: int) -> int:
    """Storage of one projection: 4-bit codes, one scale byte per 16 inputs, one f32."""
    n = out_features * in_features
    return n // 2 + n // 16 + 4


def decode_codes(words: np.ndarray, in_features: int) -> np.ndarray:
    """[out, in/8] uint32 words -> [out, in] integer codes (element 8w+n = bits 4n..4n+3)."""
    words = np.ascontiguousarray(words, dtype='<u4')
    out = words.shape[0]
    by = words.view(np.uint8).reshape(out, in_features // 2)   # byte j of word w = bits 8j..
    lo = by & 0x0F                                               # element 2j (even)
    hi = by >> 4                                                 # element 2j + 1 (odd)
    return np.stack([lo, hi], axis=-1).reshape(out, in_features)


def global_multiplier(g: np.float32, global_mode: int) -> float:
    g = np.float32(g)
    if global_mode == 0:
        return float(g)
    if global_mode == 1:
        return float(np.float32(g) / np.float32(2688.0))         # f32 division, as MLX does
    raise ValueError(global_mode)


# Values of the two elements held by one code byte: (low nibble, high nibble).
_BYTE_PAIR = np.stack([E2M1_VALUES[np.arange(256) & 0x0F], E2M1_VALUES[np.arange(256) >> 4]], axis=1)


def dequant(words: np.ndarray, scales: np.ndarray, g: np.float32, global_mode: int,
            in_features: int) -> np.ndarray:
    """Exact FP64 weights [out, in] = e2m1(code) * e4m3(scale of its 16-input block) * mult.

    Same element order as decode_codes: byte j of a row holds elements 2j (low nibble) and
    2j + 1 (high nibble).
    """
    words = np.ascontiguousarray(words, dtype='<u4')
    out = words.shape[0]
    by = words.view(np.uint8).reshape(out, in_features // 2)
    e2 = _BYTE_PAIR[by].reshape(out, in_features // 16, 16)             # [out, blocks, 16]
    sc = E4M3_VALUES[np.asarray(scales, dtype=np.uint8)]                 # [out, blocks]
    w = e2 * (sc * global_multiplier(g, global_mode))[:, :, None]
    return w.reshape(out, in_features)


def read_record(rec: np.ndarray, H: int, I: int, codes_off, scales_off, global_off,
                global_mode: int = 0):
    """Decode one expert record (uint8 bytes) into FP64 (Wg [I,H], Wu [I,H], Wd [H,I]).

    The part offsets are the bank descriptor's; the shapes are the layer's: gate and up map
    H inputs to I outputs, down maps I inputs to H outputs.
    """
    rec = np.asarray(rec, dtype=np.uint8)
    shapes = [(I, H), (I, H), (H, I)]
    mats = []
    for p, (o, i) in enumerate(shapes):
        nc, ns = o * i // 2, o * i // 16
        words = rec[codes_off[p]:codes_off[p] + nc].view('<u4').reshape(o, i // 8)
        scales = rec[scales_off[p]:scales_off[p] + ns].reshape(o, i // 16)
        g = rec[global_off[p]:global_off[p] + 4].view('<f4')[0]
        mats.append(dequant(words, scales, g, global_mode, i))
    return tuple(mats)
