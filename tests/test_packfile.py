"""Packed-layer files (host only): round trips and every check the loader makes."""
import json
import struct

import numpy as np
import pytest

import synth


@pytest.fixture(scope="module")
def msb():
    from token_top_expert_b200 import build
    build.build()
    import token_top_expert_b200 as m
    m.load_library()
    return m


@pytest.fixture(scope="module")
def layer(msb):
    w = synth.TINY.with_(d=128, inter=40, experts=3, top_e=2, rank=4)
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, w.rank)
    return w, lw, dims


def _same(a: dict, b: dict):
    assert sorted(a) == sorted(b)
    for k in a:
        assert a[k].dtype == b[k].dtype
        np.testing.assert_array_equal(a[k], b[k])


def test_round_trip_bf16_with_lowrank(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    w, lw, dims = layer
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    path = str(tmp_path / "layer.msbpack")
    packfile.save(path, dims, pk, lw.lr_a, lw.lr_b, meta={"workload": w.name, "layer": 0})
    d2, rec, pk2, a2, b2, meta = packfile.load(path, expect=dims)
    assert d2 == dims and rec == "bf16" and meta == {"workload": w.name, "layer": 0}
    _same(pk, pk2)
    np.testing.assert_array_equal(a2, lw.lr_a)
    np.testing.assert_array_equal(b2, lw.lr_b)
    # payloads start on 64-byte boundaries, after the header
    raw = open(path, "rb").read()
    assert raw[:8] == packfile.MAGIC
    hlen = struct.unpack("<I", raw[12:16])[0]
    offs = [e["offset"] for e in json.loads(raw[16:16 + hlen])["tensors"]]
    assert all(o % 64 == 0 and o >= 16 + hlen for o in offs)


def test_round_trip_q4_rank0(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    w, lw, dims = layer
    d0 = msb.Dims(dims.d, dims.inter, dims.experts, dims.top_e, 0)
    pk = msb.pack_q4(lw.gate, lw.up, lw.down, lw.router, d0)
    path = str(tmp_path / "layer_q4.msbpack")
    packfile.save(path, d0, pk, records="q4")
    d2, rec, pk2, a2, b2, _ = packfile.load(path)
    assert d2 == d0 and rec == "q4" and a2 is None and b2 is None
    _same(pk, pk2)


def _saved(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    w, lw, dims = layer
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    path = str(tmp_path / "x.msbpack")
    packfile.save(path, dims, pk, lw.lr_a, lw.lr_b)
    return path, bytearray(open(path, "rb").read())


def test_corruption_is_detected(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    path, raw = _saved(msb, layer, tmp_path)
    hlen = struct.unpack("<I", raw[12:16])[0]
    for pos in (16 + hlen + 200, len(raw) - 3):          # inside records, inside lr_b
        bad = bytearray(raw)
        bad[pos] ^= 0x10
        open(path, "wb").write(bad)
        with pytest.raises(packfile.PackFileError, match="checksum"):
            packfile.load(path)


def test_truncated_wrong_magic_version_and_dims(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    path, raw = _saved(msb, layer, tmp_path)
    _, _, dims = layer
    open(path, "wb").write(raw[:-100])
    with pytest.raises(packfile.PackFileError, match="outside the file"):
        packfile.load(path)
    open(path, "wb").write(b"NOTAPACK" + raw[8:])
    with pytest.raises(packfile.PackFileError, match="not a packed-layer file"):
        packfile.load(path)
    bad = bytearray(raw)
    bad[8:12] = struct.pack("<I", 2)
    open(path, "wb").write(bad)
    with pytest.raises(packfile.PackFileError, match="version"):
        packfile.load(path)
    open(path, "wb").write(raw)
    other = msb.Dims(dims.d, dims.inter, dims.experts, dims.top_e, dims.rank, 0)
    with pytest.raises(packfile.PackFileError, match="expected"):
        packfile.load(path, expect=other)
    assert packfile.load(path, expect=dims)[0] == dims
    # a header that does not parse
    bad = bytearray(raw)
    bad[16] = ord("#")
    open(path, "wb").write(bad)
    with pytest.raises(packfile.PackFileError, match="header"):
        packfile.load(path)


def test_save_checks_its_inputs(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    w, lw, dims = layer
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    path = str(tmp_path / "y.msbpack")
    with pytest.raises(ValueError, match="lr_a"):
        packfile.save(path, dims, pk)                              # rank 4 without factors
    short = dict(pk, alpha=pk["alpha"][:, :-1])
    with pytest.raises(ValueError, match="alpha"):
        packfile.save(path, dims, short, lw.lr_a, lw.lr_b)
    with pytest.raises(packfile.PackFileError, match="record format"):
        packfile.save(path, dims, pk, lw.lr_a, lw.lr_b, records="int3")
    assert not list(tmp_path.iterdir())                            # nothing half-written


def test_q4_file_is_not_uploaded(msb, layer, tmp_path):
    from token_top_expert_b200 import packfile
    w, lw, dims = layer
    d0 = msb.Dims(dims.d, dims.inter, dims.experts, dims.top_e, 0)
    path = str(tmp_path / "q4.msbpack")
    packfile.save(path, d0, msb.pack_q4(lw.gate, lw.up, lw.down, lw.router, d0), records="q4")
    with pytest.raises(packfile.PackFileError, match="BF16 records"):
        packfile.upload(path)          # refused before any device allocation
