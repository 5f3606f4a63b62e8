"""Seeded generators for expert banks, activations and router logits.

Every random byte of an expert record comes from a counter-based generator keyed by
(seed, layer, expert, stream), so that any single record can be regenerated on the host
without building the whole bank; ``fill.cu`` in this package writes the same bytes on the
device for banks too large to build on the host.  The generator is SplitMix64 (Steele, Lea
and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014), used in
counter mode: word i of a stream is the SplitMix64 output function applied to
key + (i + 1) * 0x9E3779B97F4A7C15 (mod 2**64).

Record layout written here (one record per expert, records ``record_stride`` bytes apart):
gate codes | up codes | down codes | gate scales | up scales | down scales | 3 x f32 global.
Gate and up are [I, H] (output rows, input columns), down is [H, I]; codes hold eight
4-bit fields per little-endian u32 word along the input axis, scales one byte per 16
inputs.  The layout is the one the bank descriptor hands to both sides; neither side
assumes it beyond the offsets it is given.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_MASK = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB

# Scale bytes are drawn uniformly over the 49 positive E4M3 encodings 0x18 (2^-4) .. 0x48 (4)
# ("config", the benchmark configurations), or over all 254 non-NaN E4M3 encodings -- zero,
# subnormals, both signs, up to 448 -- ("all_finite", range tests).
SCALE_BYTE_LO = 0x18
SCALE_BYTE_COUNT = 49
SCALE_KINDS = ("config", "all_finite")

# Record streams.
STREAM_CODES = 0
STREAM_SCALES = 1


def _mix64_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= np.uint64(_M1)
    z ^= z >> np.uint64(27)
    z *= np.uint64(_M2)
    z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, layer: int, expert: int, stream: int) -> int:
    """64-bit key of one counter stream; identical to ``moe_inputs_stream_key`` in fill.cu."""
    k = _mix64_int(seed + GOLDEN)
    for v in (layer, expert, stream):
        k = _mix64_int(k ^ ((v + GOLDEN) & _MASK))
    return k


def counter_words(key: int, n: int, start: int = 0) -> np.ndarray:
    """Words start .. start+n-1 of the stream with this key (uint64)."""
    idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    z = idx * np.uint64(GOLDEN)
    z += np.uint64(key)
    return _mix64(z)


@dataclasses.dataclass(frozen=True)
class RecordLayout:
    E: int
    H: int
    I: int
    record_bytes: int
    record_stride: int
    codes_off: tuple
    scales_off: tuple
    global_off: tuple

    @property
    def bank_bytes(self) -> int:
        return self.E * self.record_stride


def record_layout(E: int, H: int, I: int, align: int = 4096) -> RecordLayout:
    codes = I * H // 2
    scales = I * H // 16
    codes_off = (0, codes, 2 * codes)
    scales_off = (3 * codes, 3 * codes + scales, 3 * codes + 2 * scales)
    g0 = 3 * codes + 3 * scales
    global_off = (g0, g0 + 4, g0 + 8)
    rec = g0 + 12
    stride = -(-rec // align) * align
    return RecordLayout(E, H, I, rec, stride, codes_off, scales_off, global_off)


def global_value(H: int, global_mode: int = 0) -> np.float32:
    """The f32 stored as each projection's global scale.

    Mode 0 stores the multiplier itself, 1/(6*sqrt(H)).  Mode 1 stores a value g in the
    convention where the multiplier is f32(g / 2688); the value stored is f32(2688/(6*sqrt(H))).
    """
    m = 1.0 / (6.0 * math.sqrt(H))
    if global_mode == 0:
        return np.float32(m)
    return np.float32(2688.0 * m)


def record_bytes(seed: int, layer: int, expert: int, lay: RecordLayout,
                 global_mode: int = 0, scale_kind: str = "config") -> np.ndarray:
    """The lay.record_bytes bytes of record (layer, expert) as uint8 (no stride padding)."""
    out = np.empty(lay.record_bytes, dtype=np.uint8)
    n_code_bytes = 3 * lay.I * lay.H // 2
    n_scale_bytes = 3 * lay.I * lay.H // 16
    assert n_code_bytes % 8 == 0
    kc = stream_key(seed, layer, expert, STREAM_CODES)
    words = counter_words(kc, n_code_bytes // 8)
    out[0:n_code_bytes] = words.astype('<u8').view(np.uint8)
    ks = stream_key(seed, layer, expert, STREAM_SCALES)
    h = counter_words(ks, n_scale_bytes) & np.uint64(0xFFFFFFFF)
    if scale_kind == "config":
        sc = ((h * np.uint64(SCALE_BYTE_COUNT)) >> np.uint64(32)) + np.uint64(SCALE_BYTE_LO)
    elif scale_kind == "all_finite":
        i = (h * np.uint64(254)) >> np.uint64(32)            # 0 .. 253 -> 0x00..0x7E, 0x80..0xFE
        sc = np.where(i < 127, i, i + np.uint64(1))
    else:
        raise ValueError(scale_kind)
    out[n_code_bytes:n_code_bytes + n_scale_bytes] = sc.astype(np.uint8)
    g = np.full(3, global_value(lay.H, global_mode), dtype='<f4')
    out[lay.global_off[0]:lay.global_off[0] + 12] = g.view(np.uint8)
    return out


def bank_host(seed: int, layer: int, lay: RecordLayout, global_mode: int = 0,
              scale_kind: str = "config") -> np.ndarray:
    """A whole bank on the host (E * record_stride bytes, padding zero); small banks only."""
    buf = np.zeros(lay.bank_bytes, dtype=np.uint8)
    for e in range(lay.E):
        o = e * lay.record_stride
        buf[o:o + lay.record_bytes] = record_bytes(seed, layer, e, lay, global_mode, scale_kind)
    return buf


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    E: int
    k: int
    H: int
    I: int
    T: int
    layers: int = 1
    logits: str = "normal"      # "normal" | "distinct" | "zipf"
    seed: int = 0

    @property
    def layout(self) -> RecordLayout:
        return record_layout(self.E, self.H, self.I)

    def describe(self) -> str:
        return (f"E={self.E} k={self.k} H={self.H} I={self.I} T={self.T}"
                + (f" layers={self.layers}" if self.layers > 1 else "")
                + f" logits={self.logits}")


CONFIGS = {
    # Tiny layer: E=16, k=2, H=256, I=128, T=8; distinct N(0,1) logits.
    "tiny": LayerConfig("tiny", 16, 2, 256, 128, 8, 1, "distinct"),
    # Decode, batch 1: E=256, k=8, H=5120, I=2560, T=1.
    "decode_t1": LayerConfig("decode_t1", 256, 8, 5120, 2560, 1),
    # Decode, batch 64 with Zipf(s=1) expert popularity over a seeded expert permutation.
    "decode_t64_zipf": LayerConfig("decode_t64_zipf", 256, 8, 5120, 2560, 64, 1, "zipf"),
    # Prefill: T=8192, N(0,1) logits (near-balanced, ~256 rows per expert).
    "prefill_t8192": LayerConfig("prefill_t8192", 256, 8, 5120, 2560, 8192),
    # Speculative verify across depth: 24 layers, T=16 (4 streams x 4 verify rows).
    "verify24_t16": LayerConfig("verify24_t16", 256, 8, 5120, 2560, 16, 24),
}

_TAG_X, _TAG_LOGITS, _TAG_PERM, _TAG_SAMPLE, _TAG_ROT, _TAG_ACT = 1, 2, 3, 4, 5, 6


def _rng(seed: int, layer: int, tag: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, layer, tag]))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float values to BF16 (round to nearest even) and return the bit patterns."""
    import ml_dtypes
    return np.asarray(a, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def make_x(cfg: LayerConfig, seed: int | None = None, layer: int = 0) -> np.ndarray:
    """Activations [T, H] as BF16 bit patterns (uint16): N(0,1) rounded to BF16."""
    s = cfg.seed if seed is None else seed
    x = _rng(s, layer, _TAG_X).standard_normal((cfg.T, cfg.H), dtype=np.float32)
    return to_bf16_bits(x)


def make_x_wide(T: int, H: int, exps, seed: int = 0, heavy: bool = False) -> np.ndarray:
    """Activations [T, H] as BF16 bit patterns whose scale differs per token: token t is
    N(0, 1) * 2^exps[t % len(exps)] (with heavy, a standard Cauchy draw instead of N(0, 1), so
    that a few entries of a row are far larger than the rest), rounded to BF16."""
    rng = _rng(seed, 0, _TAG_X)
    base = rng.standard_cauchy((T, H)) if heavy else rng.standard_normal((T, H))
    e = np.asarray([exps[t % len(exps)] for t in range(T)], dtype=np.float64)
    v = np.clip(base * np.exp2(e)[:, None], -3.0e38, 3.0e38)
    return to_bf16_bits(v)


# Largest magnitudes the W4A4 input multipliers are set for: about the row maxima of this
# generator's x (N(0, 1) rows of a few thousand entries: ~3.8 at H = 5120) and of the mid values
# its weights give (~3 at H = 5120, I = 2560; the global scale 1/(6 sqrt(H)) keeps them similar
# across sizes), with some margin.
ACT_X_RANGE = 4.5
ACT_H_RANGE = 4.0


def make_act_scales(E: int, seed: int = 0, layer: int = 0) -> np.ndarray:
    """W4A4 input multipliers [E, 2] f32, a stand-in for a release's static activation scales:
    per expert s_x = ACT_X_RANGE 2^u / 2688 (gate/up input) and s_h = ACT_H_RANGE 2^v / 2688
    (down input), u and v uniform in [-1/4, 1/4], so that a few of the largest values saturate."""
    uv = _rng(seed, layer, _TAG_ACT).uniform(-0.25, 0.25, size=(E, 2))
    rng_ = np.array([ACT_X_RANGE, ACT_H_RANGE])[None, :]
    return (rng_ * np.exp2(uv) / 2688.0).astype(np.float32)


def make_logits(cfg: LayerConfig, seed: int | None = None, layer: int = 0,
                T: int | None = None) -> np.ndarray:
    """Router logits [T, E] f32 of the config's kind."""
    s = cfg.seed if seed is None else seed
    T = cfg.T if T is None else T
    rng = _rng(s, layer, _TAG_LOGITS)
    if cfg.logits in ("normal", "distinct"):
        lg = rng.standard_normal((T, cfg.E), dtype=np.float32)
        if cfg.logits == "distinct":
            for t in range(T):
                while len(np.unique(lg[t])) != cfg.E:
                    lg[t] = rng.standard_normal(cfg.E, dtype=np.float32)
        return lg
    if cfg.logits == "zipf":
        # Popularity p(e) proportional to 1/(1 + rank(e)), ranks a seeded permutation of the
        # experts; logit = ln p(e) + Gumbel(0, 1), so the k largest logits of a row are k
        # experts drawn without replacement in proportion to p.
        rank = _rng(s, layer, _TAG_PERM).permutation(cfg.E)
        p = 1.0 / (1.0 + rank.astype(np.float64))
        p /= p.sum()
        g = rng.gumbel(size=(T, cfg.E))
        return (np.log(p)[None, :] + g).astype(np.float32)
    raise ValueError(cfg.logits)


def sample_tokens(T: int, n: int = 512, seed: int = 0) -> np.ndarray:
    """Sorted seeded sample of min(T, n) distinct token indices."""
    if T <= n:
        return np.arange(T)
    return np.sort(np.random.default_rng(seed + 1).choice(T, n, replace=False))


def disjoint_routing_logits(E: int, k: int, sets: int, window: int, seed: int = 0) -> np.ndarray:
    """[sets, 1, E] f32 logits for one token each, such that the k largest logits of set s
    name k experts that none of the previous window-1 sets names, counting cyclically (the
    sets are used in a loop, so the last sets also avoid the experts of the first ones).

    Each row holds the same multiset as an N(0,1) draw of E values: the k largest values of
    the draw are given to k experts chosen uniformly among those not used in the window,
    the others are shuffled over the remaining experts.  Used to keep consecutive timed
    steps from re-reading expert records out of L2.
    """
    rng = _rng(seed, 0, _TAG_ROT)
    out = np.empty((sets, 1, E), dtype=np.float32)
    recent: list = []
    for s in range(sets):
        banned = set()
        for r in recent[-(window - 1):] if window > 1 else []:
            banned |= r
        wrap = set()
        for r in recent[:max(0, s + window - sets)]:      # sets 0 .. s+window-1-sets follow s cyclically
            wrap |= r
        if E - len(banned | wrap) >= k:                   # (too few experts left: window only)
            banned |= wrap
        free = np.array([e for e in range(E) if e not in banned])
        chosen = rng.choice(free, k, replace=False)
        vals = np.sort(rng.standard_normal(E).astype(np.float32))[::-1]
        while len(np.unique(vals)) != E:
            vals = np.sort(rng.standard_normal(E).astype(np.float32))[::-1]
        rest = np.array([e for e in range(E) if e not in set(chosen.tolist())])
        rng.shuffle(rest)
        row = np.empty(E, dtype=np.float32)
        row[rng.permutation(chosen)] = vals[:k]
        row[rest] = vals[k:]
        out[s, 0] = row
        recent.append(set(chosen.tolist()))
    return out
