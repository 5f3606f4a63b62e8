"""Routed-expert SwiGLU MoE layer in FP64 (oracle; test infrastructure only).

What one layer computes, for tokens t with BF16 activations x_t (taken at their exact
values) and F32 router logits l_t over E experts:
  1. route:   the k experts with the largest logits, ties to the lower expert index (a NaN
              logit ranks below -inf; -0.0 and +0.0 tie); weights w_tj = softmax over the k
              selected logits only.
  2. permute: counts[e] rows per expert, offsets = exclusive prefix sum (E + 1 entries),
              perm lists the routed rows r = t*k + j expert by expert, ascending r within an
              expert; inv[r] is the position of row r in perm.
  3. expert:  g = Wg x, u = Wu x, a = silu(g) * u with silu(g) = g / (1 + e^-g), y = Wd a.
  4. combine: out_t = sum_j w_tj * y_tj.
  5. residual (stacked layers): x_next = bf16(x + out), rounded to nearest even.

Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section
"What this pack holds" (256 routed experts, 8 active per token; activations BF16) and page
"Beam-1.0-501B-A23B VQ GGUF", section "What stays native" (router logits and SwiGLU in
FP32 in the source model; here FP64).  The pages give no router bias, no routing groups and
no clamp in SwiGLU; none is applied.

Softmax over the selected logits subtracts their maximum first; a NaN among them, or a
selected set whose maximum is infinite, yields NaN weights (IEEE propagation).
"""
from __future__ import annotations

import numpy as np

from . import encode as _encode


def route(logits: np.ndarray, k: int):
    """Top-k experts per token and their softmax weights.

    Returns ids [T, k] int64 (in rank order) and w [T, k] float64.
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    nan = np.isnan(lg)
    key = np.where(nan, 0.0, lg.astype(np.float64))
    idx = np.arange(E)
    ids = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        # np.lexsort sorts by the last key first: non-NaN before NaN, then logit descending,
        # then expert index ascending.
        order = np.lexsort((idx, -key[t], nan[t]))
        ids[t] = order[:k]
    sel = lg.astype(np.float64)[np.arange(T)[:, None], ids]
    with np.errstate(invalid="ignore", over="ignore"):
        m = sel.max(axis=1, keepdims=True)
        ex = np.exp(sel - m)
        w = ex / ex.sum(axis=1, keepdims=True)
    return ids, w


def permute(ids: np.ndarray, E: int):
    """counts [E], offsets [E+1], perm [T*k], inv [T*k] (all int64)."""
    flat = np.asarray(ids).reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return counts, offsets, perm, inv


def silu(g: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def expert_forward(Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray, X: np.ndarray) -> np.ndarray:
    """SwiGLU expert on rows X [n, H]: returns Y [n, H] (FP64)."""
    G = X @ Wg.T
    U = X @ Wu.T
    A = silu(G) * U
    return A @ Wd.T


def expert_forward_w4a4(Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray, X: np.ndarray, s_x, s_h,
                        H_rows=None):
    """The expert with NVFP4 activations (W4A4) on rows X [n, H] (exact input values): X is
    quantized with the multiplier s_x (quantize_static) before the gate and up projections; the
    mid values h = silu(g) * u, computed in FP64 from the quantized rows, are rounded to f32 (the
    precision in which they are quantized) and quantized with s_h before the down projection.
    H_rows [n, I], if given, replaces the f32 h rows (teacher forcing: a test feeds the h that
    the GPU computed).  Returns (h f32 [n, I] before quantization, Y [n, H] FP64)."""
    Xq = _encode.quantize_static(np.asarray(X, dtype=np.float32), s_x)[2]
    G = Xq @ Wg.T
    U = Xq @ Wu.T
    h = (silu(G) * U).astype(np.float32) if H_rows is None else np.asarray(H_rows, dtype=np.float32)
    hq = _encode.quantize_static(h, s_h)[2]
    return h, hq @ Wd.T


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round FP64 values to BF16 (nearest, ties to even; overflow to inf) -> uint16 bits."""
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.float32)
    fin = np.isfinite(v)
    vf = np.where(fin, v, 0.0)
    _, e = np.frexp(vf)                           # v = m * 2^e with 0.5 <= |m| < 1
    shift = np.maximum(e.astype(np.int64) - 8, -133)   # 8 significant bits; subnormal grid 2^-133
    r = np.ldexp(np.rint(np.ldexp(vf, -shift)), shift)
    big = np.abs(r) >= 2.0 ** 128
    r = np.where(big, np.copysign(np.inf, vf), r)
    out[...] = np.where(fin, r, v).astype(np.float32)
    bits = (out.view(np.uint32) >> 16).astype(np.uint16)
    bits = np.where(np.isnan(v), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


def residual_add(x_bits: np.ndarray, out_bits: np.ndarray) -> np.ndarray:
    """x_next = bf16(x + out) of two BF16 tensors (the sum is exact in FP64)."""
    return round_to_bf16_bits(bf16_bits_to_f64(x_bits) + bf16_bits_to_f64(out_bits))


def _expert_job(job):
    get_weights, e, X = job[:3]
    Wg, Wu, Wd = get_weights(e)
    if len(job) == 3:
        return expert_forward(Wg, Wu, Wd, X)
    return expert_forward_w4a4(Wg, Wu, Wd, X, *job[3:])


def layer_forward(x_bits: np.ndarray, logits: np.ndarray, k: int, get_weights,
                  tokens=None, want_rows: bool = False, map_fn=map, act_scales=None, h_rows=None):
    """One MoE layer.

    x_bits [T, H] BF16 bit patterns, logits [T, E] f32, get_weights(e) -> (Wg, Wu, Wd) FP64.
    tokens: optional list of token indices to evaluate (routing is always computed for all).
    Returns a dict with ids, w, counts, offsets, perm, inv and out [len(tokens), H] (FP64);
    with want_rows also y [len(tokens), k, H], the expert outputs before the combine.
    map_fn maps the per-expert work (decode the record, run the expert on its rows); a process
    pool's map spreads it over host cores without changing any arithmetic.
    act_scales [E, 2] f32 selects the W4A4 variant (expert_forward_w4a4): a routed row of expert e
    quantizes its token's x with the multiplier act_scales[e, 0] and its mid values with
    act_scales[e, 1]; the result then also holds h [len(tokens), k, I] (f32, before
    quantization).  h_rows [T, k, I] (optional) replaces the mid values of every routed row
    (teacher forcing).
    """
    T, E = np.asarray(logits).shape
    ids, w = route(logits, k)
    counts, offsets, perm, inv = permute(ids, E)
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    x = bf16_bits_to_f64(x_bits)
    w4a4 = act_scales is not None
    if w4a4:
        act_scales = np.asarray(act_scales, dtype=np.float32).reshape(E, 2)
    H = x.shape[1]
    y = np.zeros((len(toks), k, H))
    hs = None
    by_expert: dict = {}
    for ti, t in enumerate(toks):
        for j in range(k):
            by_expert.setdefault(int(ids[t, j]), []).append((ti, int(t), j))
    experts = sorted(by_expert)
    jobs = [(get_weights, e, x[[t for (_, t, _) in by_expert[e]]]) for e in experts]
    if w4a4:
        jobs = [job + (act_scales[e, 0], act_scales[e, 1],
                       None if h_rows is None else np.stack([h_rows[t, j] for (_, t, j) in by_expert[e]]))
                for e, job in zip(experts, jobs)]
    for e, res in zip(experts, map_fn(_expert_job, jobs)):
        Y = res
        if w4a4:
            h, Y = res
            if hs is None:
                hs = np.zeros((len(toks), k, h.shape[1]), np.float32)
            for r, (ti, _, j) in enumerate(by_expert[e]):
                hs[ti, j] = h[r]
        for r, (ti, _, j) in enumerate(by_expert[e]):
            y[ti, j] = Y[r]
    out = np.zeros((len(toks), H))
    for j in range(k):
        out += w[toks, j][:, None] * y[:, j]
    res = dict(ids=ids, w=w, counts=counts, offsets=offsets, perm=perm, inv=inv, out=out,
               tokens=toks)
    if w4a4:
        res["h"] = hs
    if want_rows:
        res["y"] = y
    return res
