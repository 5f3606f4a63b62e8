"""The GPU NVFP4 encoder against the oracle's encoder: codes, block scales and globals bit-exact
(every byte is a rounding decision both sides take in f32, nearest even), on random, heavy-tailed
and wide-range weights, exact ties, zero and tiny blocks, both global conventions, batches of
projections written into expert records, and a full-size layer encoded from BF16 weights and
run through the layer against the oracle.

Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section "What this
pack holds" (the record and the g / 2688 convention); page "Running Beam-1.0 (501B) on workstation
GPUs" (data-free NVFP4A16 quantization)."""
import numpy as np
import pytest

import moe_inputs
import oracle
from conftest import assert_layer_close
from gpu_helpers import bf16_tensor, bits_of

pytestmark = pytest.mark.gpu


def _weights(kind, n, out_f, in_f, seed):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        w = rng.standard_normal((n, out_f, in_f))
    elif kind == "cauchy":
        w = rng.standard_cauchy((n, out_f, in_f))
    elif kind == "wide":                           # rows and blocks over 2^-60 .. 2^60
        w = rng.standard_normal((n, out_f, in_f)) * 2.0 ** rng.integers(-60, 60, (n, out_f, in_f // 16)).repeat(16, 2)
    elif kind == "sparse":                         # zero blocks, zero rows, -0.0, tiny values
        w = rng.standard_normal((n, out_f, in_f))
        w[:, ::3, :] = 0.0
        w[:, 1, 16:32] = -0.0
        w[:, 2, 32:48] = 1e-35 * rng.standard_normal(16)
        w[0] = 0.0
    else:
        raise ValueError(kind)
    return moe_inputs.gen.to_bf16_bits(np.clip(w, -3e38, 3e38).astype(np.float32))


def _encode_gpu(wbits, mode, stride=None, offs=None):
    import torch
    import nvfp4_weight_only_top_b200 as moe
    n, out_f, in_f = wbits.shape
    cb, sb = out_f * in_f // 2, out_f * in_f // 16
    if offs is None:                               # scales, then codes, then the global
        offs = (((sb + 15) // 16) * 16, 0, ((sb + 15) // 16) * 16 + cb)
    co, so, go = offs
    if stride is None:
        stride = ((max(co + cb, so + sb, go + 4) + 255) // 256) * 256
    dst = torch.full(((n - 1) * stride + max(co + cb, so + sb, go + 4),), 0xA5, dtype=torch.uint8, device="cuda")
    moe.moe_nvfp4_encode(bf16_tensor(wbits.reshape(n * out_f, in_f)).view(n, out_f, in_f), dst, stride, co, so, go, mode)
    torch.cuda.synchronize()
    assert moe.moe_nvfp4_last_launch_count() == 4
    raw = dst.cpu().numpy()
    out = []
    for i in range(n):
        r = raw[i * stride:]
        codes = r[co:co + cb].view('<u4').reshape(out_f, in_f // 8)
        scales = r[so:so + sb].reshape(out_f, in_f // 16)
        g = r[go:go + 4].view('<f4')[0]
        out.append((codes.copy(), scales.copy(), np.float32(g)))
    return out


def _check(wbits, mode, **kw):
    got = _encode_gpu(wbits, mode, **kw)
    for i in range(wbits.shape[0]):
        c, s, g = oracle.encode_projection(wbits[i], mode)
        gc, gs, gg = got[i]
        assert np.array_equal(gs, s), f"projection {i}: scales differ at {np.argwhere(gs != s)[:5]}"
        assert np.array_equal(gc, oracle.pack_codes(c)), f"projection {i}: codes differ"
        assert np.float32(gg).tobytes() == np.float32(g).tobytes(), (i, gg, g)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kind", ["normal", "cauchy", "wide", "sparse"])
def test_encode_matches_the_oracle_bit_for_bit(kind, mode):
    _check(_weights(kind, 3, 40, 272, seed=len(kind) + mode), mode)


def test_encode_exact_ties_and_representable_weights():
    # every block holds a +-6 x scale x 2^-8 anchor (so the block scale is that scale exactly) and
    # ratios at every E2M1 midpoint, both signs
    rng = np.random.default_rng(9)
    n, out_f, in_f = 2, 16, 128
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.0, 6.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0], np.float64)
    w = np.zeros((n, out_f, in_f // 16, 16))
    scales = oracle.E4M3_VALUES[rng.integers(8, 0x7F, (n, out_f, in_f // 16))]
    scales[:, 0, 0] = 448.0
    for b in range(16):
        w[..., b] = rng.choice(mids, size=(n, out_f, in_f // 16)) * rng.choice([-1.0, 1.0], size=(n, out_f, in_f // 16))
    w[..., 0] = 6.0
    w = w * scales[..., None] * 2.0 ** -8
    bits = moe_inputs.gen.to_bf16_bits(w.reshape(n, out_f, in_f).astype(np.float32))
    assert np.array_equal(oracle.bf16_bits_to_f64(bits), w.reshape(n, out_f, in_f))   # exact in BF16
    _check(bits, 0)
    _check(bits, 1)


def test_encode_into_records_with_other_part_orders():
    bits = _weights("normal", 4, 24, 160, seed=3)
    cb, sb = 24 * 160 // 2, 24 * 160 // 16
    _check(bits, 0, offs=(0, cb, cb + sb + 12), stride=8192)          # codes | scales | pad | global
    _check(bits, 1, offs=(16 + sb, 16, 0), stride=4096)                # global | scales | codes


def test_encode_full_size_projections():
    """Two experts' gate projections at I=2560, H=5120 (13.1 M weights each), compared in full."""
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((2, 2560, 5120)) * np.array([0.02, 3.0])[:, None, None]).astype(np.float32)
    _check(moe_inputs.gen.to_bf16_bits(w), 0)


def test_layer_from_bf16_experts():
    """BF16 experts encoded on the GPU into a bank, then the layer on every path, against the oracle
    layer on the oracle's encoding of the same weights (identical bytes, checked first)."""
    import torch
    import nvfp4_weight_only_top_b200 as moe
    E, k, H, I, T = 16, 4, 1024, 512, 24
    rng = np.random.default_rng(12)
    gate = moe_inputs.gen.to_bf16_bits((rng.standard_normal((E, I, H)) / np.sqrt(H)).astype(np.float32))
    up = moe_inputs.gen.to_bf16_bits((rng.standard_normal((E, I, H)) / np.sqrt(H)).astype(np.float32))
    down = moe_inputs.gen.to_bf16_bits((rng.standard_normal((E, H, I)) / np.sqrt(I)).astype(np.float32))
    buf, bank = moe.encode_bank(bf16_tensor(gate.reshape(E * I, H)).view(E, I, H),
                                bf16_tensor(up.reshape(E * I, H)).view(E, I, H),
                                bf16_tensor(down.reshape(E * H, I)).view(E, H, I))
    torch.cuda.synchronize()
    lay = moe.record_layout(H, I)
    raw = buf.cpu().numpy()

    class Encoded:
        """The oracle's encoding of the same BF16 experts, decoded by the oracle (picklable)."""
        def __call__(self, e):
            rec = np.zeros(lay["record_bytes"], np.uint8)
            for p, w in enumerate((gate[e], up[e], down[e])):
                c, s, g = oracle.encode_projection(w, 0)
                pc = oracle.pack_codes(c)
                rec[lay["codes_off"][p]:lay["codes_off"][p] + pc.nbytes] = pc.view(np.uint8).reshape(-1)
                rec[lay["scales_off"][p]:lay["scales_off"][p] + s.size] = s.reshape(-1)
                rec[lay["global_off"][p]:lay["global_off"][p] + 4] = np.array([g], np.float32).view(np.uint8)
            return rec

    enc = Encoded()
    for e in (0, 7, 15):
        stride = lay["record_stride"]
        assert np.array_equal(raw[e * stride:e * stride + lay["record_bytes"]], enc(e)), f"record {e}"
    x = moe_inputs.gen.to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    src = _RecordsOf(gate, up, down, lay)
    ref = oracle.layer_forward(x, lg, k, src)["out"]
    for path in (moe.PATH_AUTO, moe.PATH_DECODE, moe.PATH_PREFILL):
        out = moe.moe_nvfp4_forward_ex(bf16_tensor(x), torch.from_numpy(lg).cuda(), bank, k, path=path)
        torch.cuda.synchronize()
        assert_layer_close(oracle.bf16_bits_to_f64(bits_of(out)), ref, f"encoded bank, path {path}")


class _RecordsOf:
    """e -> (Wg, Wu, Wd) in FP64 from the oracle's encoding of BF16 experts (picklable)."""

    def __init__(self, gate, up, down, lay):
        self.w, self.lay = (gate, up, down), lay

    def __call__(self, e):
        mats = []
        for w in self.w:
            c, s, g = oracle.encode_projection(w[e], 0)
            mats.append(oracle.dequant(oracle.pack_codes(c), s, g, 0, w.shape[2]))
        return tuple(mats)
