"""NVFP4 encoding of BF16 weights, step by step in plain numpy (oracle; test infrastructure only).

What the pages fix:
  * Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section
    "What this pack holds": a projection is stored as E2M1 codes, one E4M3 block scale per 16
    inputs and one F32 global scale; MLX takes a block's scale as e4m3(block scale) x (g / 2688)
    in f32, and the pack stores the g for which f32(g / 2688) equals the release's second-level
    (per-tensor) weight scale.  2688 = 6 x 448 is the largest E2M1 magnitude times the largest
    E4M3 magnitude.
  * Page "Running Beam-1.0 (501B) on workstation GPUs": an NVFP4A16 build quantizes the expert
    weights data-free (no calibration), keeping the activations in BF16.

The pages print no rounding rule.  The reading taken here (the plainest one that the 2688
convention supports: the per-tensor scale maps the tensor's largest magnitude onto the largest
representable product 6 x 448):
  1. amax = max |w| over the projection (exact).  The per-tensor multiplier is
     s2 = f32(amax / 2688); with global_mode 1 the stored value is g = amax itself, since
     f32(amax / 2688) is then exactly s2.  A projection of zeros stores s2 = 0 (g = 0).
  2. Per block of 16 inputs of a row: amax_b = max |w| over the block; the block scale is the
     E4M3 value nearest to f32(amax_b / f32(6 s2)), ties to even, saturating at 448.
  3. Per weight: eff = f32(e4m3(block scale) x s2); the code is the E2M1 value nearest to
     f32(w / eff), ties to even, saturating at 6, with the sign bit of w.  A block whose eff is
     0 gets magnitude code 0 for every weight (sign bit kept).
Every quotient and product above is one IEEE f32 operation (round to nearest even), because
each of them decides an integer (a scale byte or a code) and the GPU kernel takes the same
decisions in f32.  Inputs must be finite.
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import E2M1_VALUES, E4M3_VALUES

_F32 = np.float32


def _nearest_even_on_grid(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into the increasing grid of the value nearest to each a >= 0; a tie goes to the
    grid value whose last mantissa bit is 0 (the even index in both E2M1 and E4M3 magnitude
    orders); values above the top of the grid saturate to it."""
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(grid, a, side="left")          # first grid value >= a
    hi = np.minimum(hi, len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo = a - grid[lo]
    dhi = grid[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    return np.where(a >= grid[-1], len(grid) - 1, idx)


# Magnitudes in code order: E2M1 codes 0..7 and E4M3 bytes 0x00..0x7E (0x7F is NaN).
_E2M1_MAG = E2M1_VALUES[:8]
_E4M3_MAG = E4M3_VALUES[:0x7F]


def e2m1_round(r: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes of f32 values: nearest magnitude (ties to even, saturating at 6), sign
    bit from the value's sign bit."""
    r = np.asarray(r, dtype=np.float32)
    mag = _nearest_even_on_grid(np.abs(r.astype(np.float64)), _E2M1_MAG)
    return (mag | (np.signbit(r).astype(np.int64) << 3)).astype(np.uint8)


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """E4M3 (FN) bytes of non-negative f32 values: nearest (ties to even), saturating at 448."""
    v = np.asarray(v, dtype=np.float32)
    assert np.all(v >= 0)
    return _nearest_even_on_grid(v.astype(np.float64), _E4M3_MAG).astype(np.uint8)


def _global_of(w: np.ndarray):
    """(amax, s2) of f32 values: amax = max |w|, s2 = f32(amax / 2688) (0 for a zero tensor)."""
    amax = _F32(np.max(np.abs(w))) if w.size else _F32(0.0)
    s2 = _F32(amax / _F32(2688.0)) if amax > 0 else _F32(0.0)
    return amax, s2


def tensor_global(w_bits: np.ndarray):
    """(amax, s2) of a BF16 tensor: amax = max |w|, s2 = f32(amax / 2688) (0 for a zero tensor)."""
    return _global_of((np.asarray(w_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32))


def encode_projection(w_bits: np.ndarray, global_mode: int = 0):
    """Encode one projection [out, in] of BF16 weights (uint16 bit patterns).

    Returns (codes [out, in] uint8 values 0..15, scales [out, in/16] E4M3 bytes, stored global
    f32): with global_mode 0 the stored global is s2, with 1 it is g = amax.
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    return encode_f32((w_bits.astype(np.uint32) << 16).view(np.float32), global_mode)


def _encode_blocks(w: np.ndarray, s2):
    """Steps 2 and 3 for f32 values [rows, n] with a positive f32 multiplier s2 per row (an array
    broadcast over the rows): (codes [rows, n], block scale bytes [rows, n/16])."""
    rows, n = w.shape
    blocks = w.reshape(rows, n // 16, 16)
    s2 = np.asarray(s2, dtype=np.float32).reshape(-1, 1)
    amax_b = np.max(np.abs(blocks), axis=2).astype(np.float32)                  # [rows, blocks]
    denom = (_F32(6.0) * s2).astype(np.float32)
    scales = e4m3_round((amax_b / denom).astype(np.float32))                    # f32 quotient
    eff = (E4M3_VALUES[scales].astype(np.float32) * s2).astype(np.float32)      # f32 product
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (blocks / eff[:, :, None]).astype(np.float32)                       # f32 quotient
    r = np.where(eff[:, :, None] > 0, r, np.copysign(_F32(0.0), blocks))
    return e2m1_round(r).reshape(rows, n), scales


def encode_f32(w: np.ndarray, global_mode: int = 0):
    """The same encoding of f32 values [out, in] (one tensor)."""
    w = np.asarray(w, dtype=np.float32)
    out_f, in_f = w.shape
    assert in_f % 16 == 0
    assert np.all(np.isfinite(w)), "inputs must be finite"
    amax, s2 = _global_of(w)
    if s2 > 0:
        codes, scales = _encode_blocks(w, np.full(out_f, s2, np.float32))
    else:
        codes = (np.signbit(w).astype(np.uint8) << 3)
        scales = np.zeros((out_f, in_f // 16), dtype=np.uint8)
    stored = s2 if global_mode == 0 else amax
    return codes, scales, _F32(stored)


def decode_blocks(codes: np.ndarray, scales: np.ndarray, s2) -> np.ndarray:
    """Exact FP64 values e2m1(code) x e4m3(block scale) x s2 of codes [rows, n] (one value per
    byte), scale bytes [rows, n/16] and a multiplier per row (or one for all rows)."""
    codes = np.asarray(codes)
    rows, n = codes.shape
    s2 = np.broadcast_to(np.asarray(s2, dtype=np.float32).astype(np.float64).reshape(-1), (rows,))
    v = E2M1_VALUES[codes].reshape(rows, n // 16, 16) * E4M3_VALUES[np.asarray(scales)][:, :, None]
    return v.reshape(rows, n) * s2[:, None]


def quantize_rows(v: np.ndarray):
    """Each row of f32 values [rows, n] encoded on its own (the row is the tensor: its amax sets
    its multiplier s2), returned as (codes [rows, n], scales [rows, n/16], s2 [rows] f32,
    decoded values [rows, n] in FP64, exact)."""
    v = np.asarray(v, dtype=np.float32)
    rows, n = v.shape
    codes = np.empty((rows, n), np.uint8)
    scales = np.empty((rows, n // 16), np.uint8)
    g = np.empty(rows, np.float32)
    for r in range(rows):
        c, s, gg = encode_f32(v[r:r + 1], 0)
        codes[r], scales[r], g[r] = c[0], s[0], gg
    return codes, scales, g, decode_blocks(codes, scales, g)


def quantize_static(v: np.ndarray, s2):
    """NVFP4 activations with a given multiplier: rows of f32 values [rows, n] (n a multiple of
    16), each row with its positive f32 multiplier s2 (one per row, or one for all), encoded by
    steps 2 and 3 above (block scales and codes found from the values, the multiplier fixed in
    advance -- values beyond 6 x 448 x s2 saturate).  Returns (codes [rows, n], scale bytes
    [rows, n/16], decoded values [rows, n] in FP64, exact)."""
    v = np.asarray(v, dtype=np.float32)
    rows, n = v.shape
    assert n % 16 == 0
    assert np.all(np.isfinite(v)), "inputs must be finite"
    s2 = np.broadcast_to(np.asarray(s2, dtype=np.float32).reshape(-1), (rows,)).copy()
    assert np.all(s2 > 0) and np.all(np.isfinite(s2)), "multipliers must be positive and finite"
    codes, scales = _encode_blocks(v, s2)
    return codes, scales, decode_blocks(codes, scales, s2)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[out, in] codes -> [out, in/8] little-endian uint32 words (element 8w+n at bits 4n..)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out_f, in_f = codes.shape
    pairs = codes.reshape(out_f, in_f // 2, 2)
    by = (pairs[:, :, 0] | (pairs[:, :, 1] << 4)).astype(np.uint8)
    return np.ascontiguousarray(by).view('<u4').reshape(out_f, in_f // 8)
