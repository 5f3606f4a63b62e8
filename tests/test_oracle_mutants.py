"""Plants plausible mistakes in the oracle (on the CPU) and checks that its pins catch each.

Every mutant is a one-place edit of the oracle's source -- a dropped term, a wrong sign,
index, bias or operand order, a swapped role -- executed into a fresh namespace and patched
over the oracle's public names for the duration of one test.  The pins of
``test_oracle_nvfp4``, ``test_oracle_layer``, ``test_oracle_encode`` and ``test_oracle_w4a4`` are then run in order (parametrised cases
expanded) until one fails; a mutant that no pin kills fails this test.  Tests of the input
generator are skipped: they do not look at the oracle.
"""
import importlib
import inspect
import itertools
import types

import numpy as np
import pytest

import oracle
import oracle.encode
import oracle.moe
import oracle.nvfp4
import oracle.sources

PIN_MODULES = ("test_oracle_nvfp4", "test_oracle_layer", "test_oracle_encode", "test_oracle_w4a4")

# (label, oracle module, exact source text, replacement)
MUTANTS = [
    # --- E2M1 / E4M3 decoding
    ("e2m1 subnormal step 1/4", "nvfp4", "mag = 0.5 * m", "mag = 0.25 * m"),
    ("e2m1 exponent bias 0", "nvfp4", "2.0 ** (e - 1) * (1.0 + 0.5 * m)", "2.0 ** e * (1.0 + 0.5 * m)"),
    ("e2m1 mantissa weight 1", "nvfp4", "(1.0 + 0.5 * m)", "(1.0 + m)"),
    ("e2m1 sign dropped", "nvfp4", "return -mag if s else mag\n\n\ndef e4m3", "return mag\n\n\ndef e4m3"),
    ("e4m3 exponent bias 8", "nvfp4", "2.0 ** (e - 7)", "2.0 ** (e - 8)"),
    ("e4m3 subnormal scale 2^-7", "nvfp4", "2.0 ** -6 * (m / 8.0)", "2.0 ** -7 * (m / 8.0)"),
    ("e4m3 NaN pattern decoded as a number", "nvfp4", "if e == 15 and m == 7:", "if False:"),
    ("e4m3 sign dropped", "nvfp4", "(1.0 + m / 8.0)\n    return -mag if s else mag", "(1.0 + m / 8.0)\n    return mag"),
    # --- code and scale layout
    ("high nibble first (dequant)", "nvfp4",
     "np.stack([E2M1_VALUES[np.arange(256) & 0x0F], E2M1_VALUES[np.arange(256) >> 4]], axis=1)",
     "np.stack([E2M1_VALUES[np.arange(256) >> 4], E2M1_VALUES[np.arange(256) & 0x0F]], axis=1)"),
    ("high nibble first (decode_codes)", "nvfp4", "np.stack([lo, hi], axis=-1)", "np.stack([hi, lo], axis=-1)"),
    ("scale grid transposed", "nvfp4", "sc = E4M3_VALUES[np.asarray(scales, dtype=np.uint8)]",
     "sc = E4M3_VALUES[np.asarray(scales, dtype=np.uint8).T.reshape(out, in_features // 16)]"),
    ("blocks strided instead of contiguous", "nvfp4", "_BYTE_PAIR[by].reshape(out, in_features // 16, 16)",
     "_BYTE_PAIR[by].reshape(out, 16, in_features // 16).transpose(0, 2, 1)"),
    ("global scale dropped", "nvfp4", "w = e2 * (sc * global_multiplier(g, global_mode))[:, :, None]",
     "w = e2 * sc[:, :, None]"),
    ("global mode 1 divides by 448", "nvfp4", "np.float32(g) / np.float32(2688.0)", "np.float32(g) / np.float32(448.0)"),
    ("global mode 1 in f64", "nvfp4", "return float(np.float32(g) / np.float32(2688.0))", "return float(g) / 2688.0"),
    ("projection bytes: scale per 32 inputs", "nvfp4", "n // 2 + n // 16 + 4", "n // 2 + n // 32 + 4"),
    ("projection bytes: global dropped", "nvfp4", "n // 2 + n // 16 + 4", "n // 2 + n // 16"),
    # --- record parts
    ("gate and up swapped", "nvfp4", "return tuple(mats)", "return (mats[1], mats[0], mats[2])"),
    ("down read as [I, H] and transposed", "nvfp4", "mats.append(dequant(words, scales, g, global_mode, i))",
     "mats.append(dequant(words, scales, g, global_mode, i) if p < 2 else "
     "dequant(words.reshape(i, o // 8), scales.reshape(i, o // 16), g, global_mode, o).T)"),
    ("down scales from the up part", "nvfp4", "scales = rec[scales_off[p]:scales_off[p] + ns]",
     "scales = rec[scales_off[min(p, 1)]:scales_off[min(p, 1)] + ns]"),
    ("every global from the gate part", "nvfp4", "g = rec[global_off[p]:global_off[p] + 4]",
     "g = rec[global_off[0]:global_off[0] + 4]"),
    # --- routing
    ("ties to the higher index", "moe", "np.lexsort((idx, -key[t], nan[t]))", "np.lexsort((-idx, -key[t], nan[t]))"),
    ("NaN ranks highest", "moe", "np.lexsort((idx, -key[t], nan[t]))", "np.lexsort((idx, -key[t], ~nan[t]))"),
    ("smallest k selected", "moe", "np.lexsort((idx, -key[t], nan[t]))", "np.lexsort((idx, key[t], nan[t]))"),
    ("ids in expert order, not rank order", "moe", "ids[t] = order[:k]", "ids[t] = np.sort(order[:k])"),
    ("softmax denominator dropped", "moe", "w = ex / ex.sum(axis=1, keepdims=True)", "w = ex"),
    ("softmax over all E", "moe", "w = ex / ex.sum(axis=1, keepdims=True)",
     "w = ex / np.exp(lg.astype(np.float64) - m).sum(axis=1, keepdims=True)"),
    # --- permutation
    ("offsets inclusive", "moe", "offsets[1:] = np.cumsum(counts)", "offsets[:-1] = np.cumsum(counts)"),
    ("rows descending within an expert", "moe", 'perm = np.argsort(flat, kind="stable")',
     'perm = flat.size - 1 - np.argsort(flat[::-1], kind="stable")'),
    ("inv equals perm", "moe", "inv[perm] = np.arange(perm.size)", "inv[:] = perm"),
    # --- expert
    ("silu exponent sign", "moe", "g / (1.0 + np.exp(-g))", "g / (1.0 + np.exp(g))"),
    ("silu dropped", "moe", "A = silu(G) * U", "A = G * U"),
    ("silu on up instead of gate", "moe", "A = silu(G) * U", "A = silu(U) * G"),
    ("up term dropped", "moe", "A = silu(G) * U", "A = silu(G)"),
    ("up uses the gate weights", "moe", "U = X @ Wu.T", "U = X @ Wg.T"),
    ("down operand not transposed", "moe", "return A @ Wd.T", "return A @ Wd"),
    # --- combine and layer bookkeeping
    ("first weight for every slot", "moe", "out += w[toks, j][:, None] * y[:, j]", "out += w[toks, 0][:, None] * y[:, j]"),
    ("combine unweighted", "moe", "out += w[toks, j][:, None] * y[:, j]", "out += y[:, j]"),
    ("rows stored in slot 0", "moe", "y[ti, j] = Y[r]", "y[ti, 0] = Y[r]"),
    ("expert rows of the wrong token", "moe", "x[[t for (_, t, _) in by_expert[e]]]", "x[[ti for (ti, _, _) in by_expert[e]]]"),
    # --- BF16
    ("bf16 bits shifted by 15", "moe", "<< 16).view(np.float32)", "<< 15).view(np.float32)"),
    ("bf16 rounding truncates", "moe", "np.rint(np.ldexp(vf, -shift))", "np.trunc(np.ldexp(vf, -shift))"),
    ("bf16 rounding ties away from zero", "moe", "np.rint(np.ldexp(vf, -shift))",
     "(np.sign(vf) * np.floor(np.abs(np.ldexp(vf, -shift)) + 0.5))"),
    ("bf16 rounding keeps 7 bits", "moe", "e.astype(np.int64) - 8", "e.astype(np.int64) - 7"),
    ("residual drops the layer output", "moe", "round_to_bf16_bits(bf16_bits_to_f64(x_bits) + bf16_bits_to_f64(out_bits))",
     "round_to_bf16_bits(bf16_bits_to_f64(x_bits))"),
    # --- encoder
    ("rounding ties go up", "encode", "pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))", "pick_hi = dhi <= dlo"),
    ("rounding ties go to odd", "encode", "(hi % 2 == 0)", "(hi % 2 == 1)"),
    ("global over 448", "encode", "amax / _F32(2688.0)", "amax / _F32(448.0)"),
    ("global from the first element", "encode", "_F32(np.max(np.abs(w)))", "_F32(np.abs(w).reshape(-1)[0])"),
    ("block scale not divided by 6", "encode", "denom = (_F32(6.0) * s2)", "denom = (s2)"),
    ("block amax signed", "encode", "np.max(np.abs(blocks), axis=2)", "np.max(blocks, axis=2)"),
    ("block amax along rows", "encode", "amax_b = np.max(np.abs(blocks), axis=2)",
     "amax_b = np.repeat(np.max(np.abs(blocks), axis=(0, 2))[None, :], blocks.shape[0], axis=0)"),
    ("codes ignore the block scale", "encode", "r = (blocks / eff[:, :, None])", "r = (blocks / s2)"),
    ("code sign bit dropped", "encode", "(np.signbit(r).astype(np.int64) << 3)", "(0 * np.signbit(r).astype(np.int64))"),
    ("mode 1 stores the multiplier", "encode", "stored = s2 if global_mode == 0 else amax", "stored = s2"),
    ("packed high nibble first", "encode", "(pairs[:, :, 0] | (pairs[:, :, 1] << 4))", "(pairs[:, :, 1] | (pairs[:, :, 0] << 4))"),
    ("effective scale without the global", "encode", "eff = (E4M3_VALUES[scales].astype(np.float32) * s2)",
     "eff = (E4M3_VALUES[scales].astype(np.float32) * 1.0)"),
    # --- W4A4 (NVFP4 activations)
    ("W4A4 activations left unquantized", "moe", "Xq = _encode.quantize_static(np.asarray(X, dtype=np.float32), s_x)[2]",
     "Xq = X"),
    ("W4A4 mid values left unquantized", "moe", "hq = _encode.quantize_static(h, s_h)[2]", "hq = h.astype(np.float64)"),
    ("W4A4 down input with the gate/up multiplier", "moe", "act_scales[e, 0], act_scales[e, 1],",
     "act_scales[e, 0], act_scales[e, 0],"),
    ("W4A4 multipliers by slot instead of expert", "moe", "act_scales[e, 0], act_scales[e, 1],",
     "act_scales[0, 0], act_scales[0, 1],"),
    ("W4A4 teacher forcing ignored", "moe", "None if h_rows is None else np.stack(", "None if True else np.stack("),
    ("static multiplier of another row", "encode", "(rows,)).copy()\n    assert np.all(s2 > 0)",
     "(rows,))[::-1].copy()\n    assert np.all(s2 > 0)"),
    ("static quantizer decodes without the multiplier", "encode", "return v.reshape(rows, n) * s2[:, None]",
     "return v.reshape(rows, n)"),
    ("static scale divides by 448", "encode", "denom = (_F32(6.0) * s2)", "denom = (_F32(448.0) * s2)"),
]


def _pin_cases():
    cases = []
    for modname in PIN_MODULES:
        mod = importlib.import_module(modname)
        for name, fn in vars(mod).items():
            if not name.startswith("test_") or not callable(fn) or name.startswith("test_generator_"):
                continue
            grids = []
            for m in getattr(fn, "pytestmark", []):
                if m.name != "parametrize":
                    continue
                names = [s.strip() for s in m.args[0].split(",")] if isinstance(m.args[0], str) else list(m.args[0])
                grids.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in m.args[1]])
            for combo in itertools.product(*grids):
                kw = {k: v for d in combo for k, v in d.items()}
                assert set(kw) == set(inspect.signature(fn).parameters), name
                cases.append((f"{modname}.{name}{kw or ''}", fn, kw))
    return cases


def _run_pins():
    """Names of the pins that fail, stopping at the first."""
    for label, fn, kw in _pin_cases():
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except Exception as exc:  # noqa: BLE001 -- an assertion or any error kills the mutant
            return f"{label}: {type(exc).__name__}"
    return None


def _apply(mp, modname, old, new):
    real = getattr(oracle, modname)
    src = inspect.getsource(real)
    assert src.count(old) >= 1, f"mutation site not found in oracle.{modname}: {old!r}"
    ns = types.ModuleType(real.__name__ + "_mutant")
    ns.__dict__.update(__package__="oracle", __file__=real.__file__)
    exec(compile(src.replace(old, new, 1), real.__file__, "exec"), ns.__dict__)
    for name, value in vars(ns).items():
        if name.startswith("__") or not hasattr(real, name) or inspect.ismodule(value):
            continue
        orig = getattr(real, name)
        mp.setattr(real, name, value)
        for holder in (oracle, oracle.sources):
            if getattr(holder, name, None) is orig:
                mp.setattr(holder, name, value)


def test_harness_runs_every_pin_clean():
    cases = _pin_cases()
    assert len(cases) >= 30
    assert _run_pins() is None


@pytest.mark.parametrize("label,modname,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_killed(label, modname, old, new, monkeypatch):
    _apply(monkeypatch, modname, old, new)
    killed_by = _run_pins()
    assert killed_by is not None, f"no pin catches the planted mistake: {label}"
