"""Weights in from safetensors checkpoints (host only): a small Qwen3-MoE-named model
written with the safetensors library, read back by the package's own reader."""
import os

import numpy as np
import pytest
import torch
from safetensors.torch import save_file

import synth


@pytest.fixture(scope="module")
def msb():
    from token_top_expert_b200 import build
    build.build()
    import token_top_expert_b200 as m
    m.load_library()
    return m


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _model(tmp_path, dtype="bf16"):
    """Layer 0 dense (no router), layer 1 a sparse-MoE block (E = 3, I = 40, d = 64),
    split over two shards, plus tensors the reader must ignore.  Returns the workload,
    the layer's expected BF16 bits (model layout) and the shard paths."""
    w = synth.TINY.with_(d=64, inter=40, experts=3, top_e=2, rank=0)
    lw = synth.layer_weights(w)
    if dtype == "f32":
        rng = np.random.default_rng(0)
        src = {k: rng.normal(0, 0.02, getattr(lw, k).shape).astype(np.float32)
               for k in ("gate", "up", "down", "router")}
        for k, v in src.items():
            setattr(lw, k, synth.f32_to_bf16_bits(v))
        mk = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    else:
        src = {k: getattr(lw, k) for k in ("gate", "up", "down", "router")}
        mk = _bf16_tensor
    zeros = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)  # noqa: E731
    shard_a = {"model.embed_tokens.weight": zeros(10, 64),
               "model.layers.0.mlp.gate_proj.weight": zeros(40, 64),
               "model.layers.1.self_attn.q_proj.weight": zeros(64, 64),
               "model.layers.1.mlp.gate.weight": mk(src["router"].T)}
    shard_b = {}
    for e in range(w.experts):
        dst = shard_a if e < 2 else shard_b
        p = "model.layers.1.mlp.experts.%d." % e
        dst[p + "gate_proj.weight"] = mk(src["gate"][e])
        dst[p + "up_proj.weight"] = mk(src["up"][e])
        dst[p + "down_proj.weight"] = mk(src["down"][e])
    paths = [str(tmp_path / "model-00001-of-00002.safetensors"),
             str(tmp_path / "model-00002-of-00002.safetensors")]
    save_file(shard_a, paths[0])
    save_file(shard_b, paths[1])
    return w, lw, paths


def test_reads_a_bf16_layer_bit_for_bit(msb, tmp_path):
    from token_top_expert_b200 import checkpoint
    w, lw, paths = _model(tmp_path)
    sh = checkpoint.Shards(paths)
    assert checkpoint.moe_layers(sh) == [1]
    gate, up, down, router = checkpoint.layer_weights(sh, 1)
    for a, b in ((gate, lw.gate), (up, lw.up), (down, lw.down), (router, lw.router)):
        assert a.dtype == np.uint16
        np.testing.assert_array_equal(a, b)
    dims, packed, a, b = checkpoint.pack_layer(sh, 1, top_e=2)
    assert (dims.d, dims.inter, dims.experts, dims.top_e, dims.rank) == (64, 40, 3, 2, 0)
    ref = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    for k in ref:
        np.testing.assert_array_equal(packed[k], ref[k])
    assert a is None and b is None


def test_f32_checkpoint_is_rounded_to_bf16(msb, tmp_path):
    from token_top_expert_b200 import checkpoint
    w, lw, paths = _model(tmp_path, dtype="f32")
    gate, up, down, router = checkpoint.layer_weights(checkpoint.Shards(paths), 1)
    # synth's float32 -> BF16 rounding is an independent nearest-even implementation
    for a, b in ((gate, lw.gate), (up, lw.up), (down, lw.down), (router, lw.router)):
        np.testing.assert_array_equal(a, b)


def test_pack_layer_with_derived_factors_and_q4(msb, tmp_path):
    from token_top_expert_b200 import checkpoint, lowrank
    w, lw, paths = _model(tmp_path)
    sh = checkpoint.Shards(paths)
    dims, packed, a, b = checkpoint.pack_layer(sh, 1, top_e=2, rank=4, k=12, lowrank_samples=256)
    a0, b0 = lowrank.derive_lowrank(lw.gate, lw.up, lw.down, k=12, rank=4, samples=256)
    np.testing.assert_array_equal(a, a0)
    np.testing.assert_array_equal(b, b0)
    d0, pq, _, _ = checkpoint.pack_layer(sh, 1, top_e=2, records="q4")
    ref = msb.pack_q4(lw.gate, lw.up, lw.down, lw.router, d0)
    np.testing.assert_array_equal(pq["records"], ref["records"])
    with pytest.raises(ValueError, match="budget"):
        checkpoint.pack_layer(sh, 1, top_e=2, rank=4)


def test_missing_or_malformed_tensors_are_reported(msb, tmp_path):
    from token_top_expert_b200 import checkpoint
    w, lw, paths = _model(tmp_path)
    with pytest.raises(checkpoint.CheckpointError, match="experts.2"):
        checkpoint.layer_weights(checkpoint.Shards(paths[:1]), 1)     # second shard missing
    with pytest.raises(checkpoint.CheckpointError, match="not found"):
        checkpoint.layer_weights(checkpoint.Shards(paths), 0)         # dense layer
    bad = {"model.layers.1.mlp.gate.weight": _bf16_tensor(lw.router.T),
           "model.layers.1.mlp.experts.0.gate_proj.weight": _bf16_tensor(lw.gate[0]),
           "model.layers.1.mlp.experts.0.up_proj.weight": _bf16_tensor(lw.up[0][:, :32])}
    p = str(tmp_path / "bad.safetensors")
    save_file(bad, p)
    with pytest.raises(checkpoint.CheckpointError, match="shape"):
        checkpoint.layer_weights(checkpoint.Shards(p), 1)
    raw = open(paths[0], "rb").read()
    open(p, "wb").write(raw[:20])
    with pytest.raises(checkpoint.CheckpointError):
        checkpoint.Shards(p)


def test_prepare_writes_one_checked_file_per_moe_layer(msb, tmp_path):
    from token_top_expert_b200 import checkpoint, packfile, prepare
    w, lw, paths = _model(tmp_path)
    out = tmp_path / "packed"
    assert prepare.main(["--out", str(out), "--top-e", "2", "--rank", "4", "--k", "12",
                         "--lowrank-samples", "256"] + paths) == 0
    assert sorted(os.listdir(out)) == ["layer_001.msbpack"]
    dims, rec, packed, a, b, meta = packfile.load(str(out / "layer_001.msbpack"))
    assert meta == {"shards": [os.path.basename(p) for p in paths], "layer": 1, "k": 12}
    d0, p0, a0, b0 = checkpoint.pack_layer(checkpoint.Shards(paths), 1, top_e=2, rank=4, k=12,
                                           lowrank_samples=256)
    assert dims == d0 and rec == "bf16"
    for k in p0:
        np.testing.assert_array_equal(packed[k], p0[k])
    np.testing.assert_array_equal(a, a0)
    np.testing.assert_array_equal(b, b0)
    with pytest.raises(SystemExit):
        prepare.main(["--out", str(out), "--top-e", "2", "--rank", "4"] + paths)   # no --k
