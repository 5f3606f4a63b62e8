"""Streaming packs on the host (no GPU): the manifest reader, the record geometry, the sha256 check
of every record against the manifest (the page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts /
MLX 8-bit residents", section "What this pack holds": offset, length and sha256 per record, 4 KiB
record alignment, the 9 parts of a record), and the loader's refusals of malformed packs."""
import hashlib
import json
import os

import numpy as np
import pytest

import moe_inputs
from moe_inputs import pack as mpack
import nvfp4_weight_only_top_b200 as moe
from nvfp4_weight_only_top_b200 import _abi


@pytest.mark.parametrize("n", list(range(0, 130)) + [1000, 4096, 65537])
def test_sha256_matches_hashlib(n):
    d = np.random.default_rng(n).integers(0, 256, n, dtype=np.uint8).tobytes()
    assert moe.moe_nvfp4_sha256(d) == hashlib.sha256(d).digest()


@pytest.fixture(scope="module")
def small_pack(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("pack"))
    man = mpack.write_pack(d, layers=3, E=4, H=256, I=128, seed=5,
                           inexact=[(1, 2, "down"), (0, 0, "gate")])
    return d, man


def test_open_reads_the_geometry(small_pack):
    d, man = small_pack
    p = moe.Pack(os.path.join(d, "expert-manifest.json"))
    i = p.info
    lay = moe_inputs.record_layout(4, 256, 128)
    assert (i["layers"], i["experts"], i["hidden"], i["intermediate"]) == (3, 4, 256, 128)
    assert i["record_bytes"] == lay.record_bytes and i["record_stride"] == lay.record_stride
    assert i["record_stride"] % 4096 == 0
    assert tuple(i["codes_off"]) == lay.codes_off and tuple(i["scales_off"]) == lay.scales_off
    assert tuple(i["global_off"]) == lay.global_off
    assert i["global_mode"] == 1 and i["inexact_globals"] == 2
    assert p.verify() == 0 and p.verify(layer=2, threads=1) == 0
    p.close()


def test_verify_finds_a_corrupted_record(tmp_path):
    mpack.write_pack(str(tmp_path), layers=2, E=3, H=256, I=128, seed=1, corrupt=[(1, 2)])
    p = moe.Pack(str(tmp_path / "expert-manifest.json"))
    assert p.verify(layer=0) == 0
    with pytest.raises(moe.MoeError) as ei:
        p.verify()
    assert ei.value.code == _abi.ERR_INTEGRITY and "1 bad" in str(ei.value)
    p.close()


def _rewrite(path, fn):
    m = json.load(open(path))
    fn(m)
    json.dump(m, open(path, "w"))


@pytest.mark.parametrize("edit,code", [
    (lambda m: m.update(format="other-format"), _abi.ERR_INVALID_ARG),
    (lambda m: m.update(layout="nvfp4-other"), _abi.ERR_INVALID_ARG),
    (lambda m: m["parts"].pop(), _abi.ERR_INVALID_ARG),                          # 8 parts
    (lambda m: m["parts"][0].update(length=m["parts"][0]["length"] - 16), _abi.ERR_INVALID_ARG),
    (lambda m: m["parts"][1].update(name="gate.codes"), _abi.ERR_INVALID_ARG),     # repeated part
    (lambda m: m["parts"][3].update(offset=m["parts"][3]["offset"] + 8), _abi.ERR_INVALID_ARG),
    (lambda m: m["records"][2].update(offset=m["records"][2]["offset"] + 512), _abi.ERR_INVALID_ARG),
    (lambda m: m["records"].pop(), _abi.ERR_INVALID_ARG),                        # a record missing
    (lambda m: m["records"][0].update(sha256="xyz"), _abi.ERR_INVALID_ARG),
    (lambda m: m["records"][-1].update(offset=m["records"][-1]["offset"] + 4096 * 64), _abi.ERR_IO),
    (lambda m: m.update(hidden=512), _abi.ERR_INVALID_ARG),                       # parts no longer fit
])
def test_open_refuses_malformed_manifests(tmp_path, edit, code):
    mpack.write_pack(str(tmp_path), layers=1, E=3, H=256, I=128)
    _rewrite(str(tmp_path / "expert-manifest.json"), edit)
    with pytest.raises(moe.MoeError) as ei:
        moe.Pack(str(tmp_path / "expert-manifest.json"))
    assert ei.value.code == code


def test_open_refuses_broken_json_and_missing_files(tmp_path):
    mpack.write_pack(str(tmp_path), layers=1, E=2, H=256, I=128)
    man = tmp_path / "expert-manifest.json"
    with pytest.raises(moe.MoeError) as ei:
        moe.Pack(str(man), str(tmp_path / "nope.bin"))
    assert ei.value.code == _abi.ERR_IO
    man.write_text(man.read_text()[:-20])
    with pytest.raises(moe.MoeError) as ei:
        moe.Pack(str(man))
    assert ei.value.code == _abi.ERR_INVALID_ARG and "manifest" in str(ei.value)


def test_pack_records_are_the_generators_bytes(small_pack):
    d, _ = small_pack
    lay = moe_inputs.record_layout(4, 256, 128)
    for (l, e) in [(0, 0), (2, 3), (1, 1)]:
        assert np.array_equal(mpack.pack_record(d, l, e), moe_inputs.record_bytes(5, l, e, lay, global_mode=1))


def test_load_without_a_device_is_unsupported(small_pack):
    d, _ = small_pack
    p = moe.Pack(os.path.join(d, "expert-manifest.json"))
    lib = moe.lib()
    rc = lib.moe_nvfp4_pack_load(p.handle, 0, None, 0, None, p.info["record_stride"], 0, None)
    assert rc == _abi.ERR_UNSUPPORTED
    assert lib.moe_nvfp4_pack_load(p.handle, 7, None, 0, None, p.info["record_stride"], 0, None) == _abi.ERR_INVALID_ARG
    assert lib.moe_nvfp4_pack_load(p.handle, 0, None, 0, None, 16, 0, None) == _abi.ERR_INVALID_ARG
    p.close()
