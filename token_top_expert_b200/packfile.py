"""Packed-layer files: the host packer's output saved once and reloaded with checks.

Packing a layer (ternary sketch, channel records) is offline work; a file keeps its
result so that a process can upload a layer without packing it again.  Loading verifies
everything it depends on and raises ``PackFileError`` on any mismatch instead of handing
back wrong weights.

File layout (little-endian):

    8 bytes   magic b"MSBPACK\\0"
    4 bytes   format version (1)
    4 bytes   header length H
    H bytes   UTF-8 JSON header: {"dims": {d, inter, experts, top_e, rank, renorm},
              "records": "bf16" | "q4", "meta": {...},
              "tensors": [{"name", "dtype", "shape", "offset", "nbytes", "crc32"}, ...]}
    payload   each tensor's bytes at its offset (a multiple of 64 from the file start)

Tensors: records, sketch, alpha, router_t (as returned by ``pack`` or ``pack_q4``) and,
with rank > 0, lr_a [E][d][r] and lr_b [E][r][d] (BF16 bits).  The expected shape of
every tensor follows from the dims (the sketch size and record size are asked of
libmsb, so the file and the kernels agree on them).
"""
from __future__ import annotations

import ctypes
import json
import os
import struct
import zlib

import numpy as np

from . import _lib
from .block import Dims, PackedLayer

MAGIC = b"MSBPACK\0"
VERSION = 1
_ALIGN = 64
_DTYPES = {"uint16": np.uint16, "uint32": np.uint32, "float32": np.float32, "uint8": np.uint8}


class PackFileError(ValueError):
    """The file is not a packed layer this library can use (format, dims, size, checksum)."""


def _expected(dims: Dims, records: str) -> dict:
    lib = _lib.load()
    cd = dims.c()
    words = lib.msb_sketch_words(ctypes.byref(cd))
    if words == 0:
        raise PackFileError("dims rejected by the library: %s" % (dims,))
    E, I, d, r = dims.experts, dims.inter, dims.d, dims.rank
    if records == "bf16":
        rec = ((E, I, 3 * d), "uint16")
    elif records == "q4":
        rec = ((E, I, lib.msb_q4_record_bytes(ctypes.byref(cd))), "uint8")
    else:
        raise PackFileError("unknown record format %r" % (records,))
    shapes = {"records": rec, "sketch": ((words,), "uint32"), "alpha": ((E, dims.ipad), "float32"),
              "router_t": ((E, d), "uint16")}
    if r > 0:
        shapes["lr_a"] = ((E, d, r), "uint16")
        shapes["lr_b"] = ((E, r, d), "uint16")
    return shapes


def save(path: str, dims: Dims, packed: dict, lr_a: np.ndarray | None = None,
         lr_b: np.ndarray | None = None, records: str = "bf16", meta: dict | None = None) -> None:
    """Write a packed layer.  packed: the dict ``pack``/``pack_q4`` returned; lr_a/lr_b:
    BF16 bits, required when dims.rank > 0; meta: free JSON-serialisable provenance
    (workload name, seed, layer, ...).  The file is written to a temporary name and
    renamed, so a reader never sees a partial file."""
    shapes = _expected(dims, records)
    arrays = dict(packed)
    if dims.rank > 0:
        if lr_a is None or lr_b is None:
            raise ValueError("rank %d needs lr_a and lr_b" % dims.rank)
        arrays["lr_a"], arrays["lr_b"] = lr_a, lr_b
    entries, views = [], []
    for name, (shape, dtype) in shapes.items():
        a = np.ascontiguousarray(arrays[name])
        if a.shape != tuple(shape) or a.dtype != _DTYPES[dtype]:
            raise ValueError("%s: expected %s %s, got %s %s" % (name, dtype, shape, a.dtype, a.shape))
        v = memoryview(a).cast("B")
        entries.append({"name": name, "dtype": dtype, "shape": list(shape), "nbytes": v.nbytes,
                        "crc32": zlib.crc32(v)})
        views.append(v)
    header = {"dims": {"d": dims.d, "inter": dims.inter, "experts": dims.experts,
                       "top_e": dims.top_e, "rank": dims.rank, "renorm": dims.renorm},
              "records": records, "meta": meta or {}, "tensors": entries}
    # the offsets depend on the header's length and the length on the offsets' digits:
    # measure the header with placeholders at least as wide, then pad it to that length
    for e in entries:
        e["offset"] = 10 ** 15
    hlen = len(json.dumps(header).encode())
    offset = (16 + hlen + _ALIGN - 1) // _ALIGN * _ALIGN
    for e in entries:
        e["offset"] = offset
        offset = (offset + e["nbytes"] + _ALIGN - 1) // _ALIGN * _ALIGN
    text = json.dumps(header).encode()
    text += b" " * (hlen - len(text))
    tmp = path + ".tmp%d" % os.getpid()
    try:
        with open(tmp, "wb") as f:
            f.write(MAGIC + struct.pack("<II", VERSION, len(text)) + text)
            for e, v in zip(entries, views):
                f.write(b"\0" * (e["offset"] - f.tell()))
                f.write(v)
        os.replace(tmp, path)
    except BaseException:
        if os.path.exists(tmp):
            os.remove(tmp)
        raise


def load(path: str, expect: Dims | None = None):
    """Read and verify a packed layer.  Returns (dims, records format, packed dict, lr_a,
    lr_b, meta).  With ``expect``, the file's dims must equal it.  Raises PackFileError
    on a wrong magic or version, dims the library rejects or that differ from
    ``expect``, a tensor of the wrong shape or type, a truncated file or a checksum
    mismatch."""
    with open(path, "rb") as f:
        f.seek(0, os.SEEK_END)
        size = f.tell()
        f.seek(0)
        head = f.read(16)
        if len(head) < 16 or head[:8] != MAGIC:
            raise PackFileError("%s: not a packed-layer file" % path)
        version, hlen = struct.unpack("<II", head[8:16])
        if version != VERSION:
            raise PackFileError("%s: format version %d, this library reads %d"
                                % (path, version, VERSION))
        try:
            header = json.loads(f.read(hlen).decode())
            hd = header["dims"]
            dims = Dims(int(hd["d"]), int(hd["inter"]), int(hd["experts"]), int(hd["top_e"]),
                        int(hd["rank"]), int(hd["renorm"]))
            records = header["records"]
            entries = {e["name"]: e for e in header["tensors"]}
        except (ValueError, KeyError, TypeError) as exc:
            raise PackFileError("%s: unreadable header (%s)" % (path, exc)) from None
        if expect is not None and dims != expect:
            raise PackFileError("%s: dims %s, expected %s" % (path, dims, expect))
        shapes = _expected(dims, records)
        if set(entries) != set(shapes):
            raise PackFileError("%s: tensors %s, expected %s"
                                % (path, sorted(entries), sorted(shapes)))
        out = {}
        for name, (shape, dtype) in shapes.items():
            e = entries[name]
            try:
                if list(e["shape"]) != list(shape) or e["dtype"] != dtype:
                    raise PackFileError("%s: %s is %s %s, expected %s %s"
                                        % (path, name, e["dtype"], e["shape"], dtype, list(shape)))
                lo, stored, crc = int(e["offset"]), int(e["nbytes"]), int(e["crc32"])
            except (KeyError, TypeError, ValueError) as exc:
                if isinstance(exc, PackFileError):
                    raise
                raise PackFileError("%s: unreadable entry for %s (%s)" % (path, name, exc)) from None
            nbytes = int(np.prod(shape)) * np.dtype(_DTYPES[dtype]).itemsize
            if stored != nbytes or lo < 16 + hlen or lo + nbytes > size:
                raise PackFileError("%s: %s lies outside the file (truncated?)" % (path, name))
            f.seek(lo)
            a = np.empty(shape, _DTYPES[dtype])
            if f.readinto(memoryview(a).cast("B")) != nbytes:
                raise PackFileError("%s: short read of %s" % (path, name))
            if zlib.crc32(memoryview(a).cast("B")) != crc:
                raise PackFileError("%s: checksum mismatch in %s" % (path, name))
            out[name] = a
    lr_a, lr_b = out.pop("lr_a", None), out.pop("lr_b", None)
    return dims, records, out, lr_a, lr_b, header.get("meta", {})


def upload(path: str, expect: Dims | None = None, device="cuda") -> PackedLayer:
    """Load, verify and upload a packed layer with BF16 records (the kernels read no
    4-bit records, so a 4-bit file is refused)."""
    dims, records, packed, lr_a, lr_b, _ = load(path, expect)
    if records != "bf16":
        raise PackFileError("%s: %s records cannot be uploaded: the block's kernels read "
                            "BF16 records" % (path, records))
    return PackedLayer.from_host(dims, packed, lr_a, lr_b, device)
