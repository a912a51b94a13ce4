"""Weights in from safetensors checkpoints of Qwen3-MoE-style models (host only).

The block needs nothing but the model's weights ("A reader built from weights alone"):
this module reads one sparse-MoE layer's router and expert matrices from the shards of a
checkpoint, in the tensor naming of Qwen3-MoE-style checkpoints,

    {prefix}.{l}.mlp.gate.weight                    router   [E][d]
    {prefix}.{l}.mlp.experts.{e}.gate_proj.weight   W_gate   [I][d]
    {prefix}.{l}.mlp.experts.{e}.up_proj.weight     W_up     [I][d]
    {prefix}.{l}.mlp.experts.{e}.down_proj.weight   W_down   [d][I]

(prefix "model.layers"), and returns them in the model layout the packer takes
(``pack`` / ``pack_q4``): gate, up [E][I][d], down [E][d][I], router [d][E], BF16 bits.

Files are read with a small reader of the safetensors layout (an 8-byte little-endian
header length, a JSON header of {name: {dtype, shape, data_offsets}}, then the data),
memory-mapped, so BF16 tensors arrive as their 16-bit patterns without conversion; F32
and F16 tensors are rounded to BF16 (nearest, ties to even).
"""
from __future__ import annotations

import json
import os
import re
import struct

import numpy as np

from .block import Dims
from .lowrank import _bf16_bits

_NP = {"BF16": np.uint16, "F16": np.float16, "F32": np.float32}


class CheckpointError(ValueError):
    """A tensor is missing, has an unexpected shape or dtype, or a file is malformed."""


class Shards:
    """Index of the tensors in one or more .safetensors files (memory-mapped on read)."""

    def __init__(self, paths):
        if isinstance(paths, (str, os.PathLike)):
            paths = [paths]
        self.where = {}
        for path in paths:
            path = os.fspath(path)
            with open(path, "rb") as f:
                raw = f.read(8)
                if len(raw) != 8:
                    raise CheckpointError("%s: not a safetensors file" % path)
                (n,) = struct.unpack("<Q", raw)
                size = os.fstat(f.fileno()).st_size
                if n > size - 8:
                    raise CheckpointError("%s: header length %d beyond the file" % (path, n))
                try:
                    header = json.loads(f.read(n))
                except ValueError as exc:
                    raise CheckpointError("%s: unreadable header (%s)" % (path, exc)) from None
            base = 8 + n
            for name, info in header.items():
                if name == "__metadata__":
                    continue
                lo, hi = info["data_offsets"]
                if not 0 <= lo <= hi <= size - base:
                    raise CheckpointError("%s: %s lies outside the file" % (path, name))
                self.where[name] = (path, info["dtype"], tuple(info["shape"]), base + lo, hi - lo)

    def names(self):
        return self.where.keys()

    def bf16(self, name: str, shape=None) -> np.ndarray:
        """Tensor `name` as BF16 bits (uint16), checked against `shape` if given."""
        if name not in self.where:
            raise CheckpointError("tensor %s not found" % name)
        path, dtype, shp, off, nbytes = self.where[name]
        if dtype not in _NP:
            raise CheckpointError("%s: dtype %s (expected BF16, F16 or F32)" % (name, dtype))
        if shape is not None and shp != tuple(shape):
            raise CheckpointError("%s: shape %s, expected %s" % (name, shp, tuple(shape)))
        n = int(np.prod(shp)) if shp else 1
        if n * np.dtype(_NP[dtype]).itemsize != nbytes:
            raise CheckpointError("%s: %d bytes for shape %s %s" % (name, nbytes, shp, dtype))
        a = np.memmap(path, dtype=_NP[dtype], mode="r", offset=off, shape=shp)
        if dtype == "BF16":
            return np.array(a)
        return _bf16_bits(np.asarray(a, dtype=np.float32)).reshape(shp)


def moe_layers(shards: Shards, prefix: str = "model.layers") -> list:
    """Indices of the layers that have a sparse-MoE block (a router tensor)."""
    pat = re.compile(r"^%s\.(\d+)\.mlp\.gate\.weight$" % re.escape(prefix))
    return sorted(int(m.group(1)) for m in map(pat.match, shards.names()) if m)


def layer_weights(shards: Shards, layer: int, prefix: str = "model.layers"):
    """One MoE layer in the packer's model layout: (gate [E][I][d], up [E][I][d],
    down [E][d][I], router [d][E]) as BF16 bits.  E, I and d come from the router and
    the first expert; every expert must be present with the same shapes."""
    p = "%s.%d.mlp" % (prefix, layer)
    router = shards.bf16(p + ".gate.weight")
    if router.ndim != 2:
        raise CheckpointError("%s.gate.weight: shape %s, expected [E][d]" % (p, router.shape))
    E, d = router.shape
    g0 = shards.bf16(p + ".experts.0.gate_proj.weight")
    if g0.ndim != 2 or g0.shape[1] != d:
        raise CheckpointError("%s.experts.0.gate_proj.weight: shape %s, expected [I][%d]"
                              % (p, g0.shape, d))
    I = g0.shape[0]
    gate = np.empty((E, I, d), np.uint16)
    up = np.empty((E, I, d), np.uint16)
    down = np.empty((E, d, I), np.uint16)
    for e in range(E):
        q = "%s.experts.%d." % (p, e)
        gate[e] = g0 if e == 0 else shards.bf16(q + "gate_proj.weight", (I, d))
        up[e] = shards.bf16(q + "up_proj.weight", (I, d))
        down[e] = shards.bf16(q + "down_proj.weight", (d, I))
    return gate, up, down, np.ascontiguousarray(router.T)


def pack_layer(shards: Shards, layer: int, top_e: int, rank: int = 0, k: int | None = None,
               renorm: int = 1, records: str = "bf16", prefix: str = "model.layers",
               lowrank_samples: int = 4096):
    """Read, pack and (with rank > 0) derive the compensation factors of one MoE layer.

    top_e: the model's routed experts per token; rank: compensation rank r (0: none);
    k: the channel budget the factors are derived for (required when rank > 0);
    records: "bf16" (the kernels' records) or "q4" (4-bit records).
    Returns (dims, packed dict, lr_a, lr_b), ready for ``packfile.save`` or
    ``PackedLayer.from_host``."""
    from . import block, lowrank
    gate, up, down, router = layer_weights(shards, layer, prefix)
    E, I, d = gate.shape
    dims = Dims(d, I, E, top_e, rank, renorm)
    packer = {"bf16": block.pack, "q4": block.pack_q4}.get(records)
    if packer is None:
        raise ValueError("records must be 'bf16' or 'q4'")
    packed = packer(gate, up, down, router, dims)
    lr_a = lr_b = None
    if rank > 0:
        if k is None:
            raise ValueError("rank > 0 needs the channel budget k the factors compensate")
        lr_a, lr_b = lowrank.derive_lowrank(gate, up, down, k=k, rank=rank,
                                            samples=lowrank_samples)
    return dims, packed, lr_a, lr_b
