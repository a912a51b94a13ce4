"""Python binding of libmsb: argument marshalling over the C ABI, nothing else.

PyTorch provides device memory and streams; every step of the block runs in
libmsb's CUDA kernels.  Host-side packing calls libmsb's C++ packer.
"""
from __future__ import annotations

import ctypes
import dataclasses

import numpy as np

from . import _lib
from ._lib import MsbDims, MsbError, MsbTrace


@dataclasses.dataclass(frozen=True)
class Dims:
    d: int
    inter: int
    experts: int
    top_e: int
    rank: int
    renorm: int = 1

    @property
    def ipad(self) -> int:
        return (self.inter + 15) // 16 * 16

    def c(self) -> MsbDims:
        return MsbDims(self.d, self.inter, self.experts, self.top_e, self.rank, self.renorm)


def _ptr(a) -> int:
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def _check(rc: int, what: str):
    if rc != _lib.MSB_OK:
        raise MsbError(rc, what)


# ------------------------------------------------------------------ packing (host)

def sketch_words(dims: Dims) -> int:
    return _lib.load().msb_sketch_words(ctypes.byref(dims.c()))


def q4_record_bytes(dims: Dims) -> int:
    """Bytes of one 4-bit channel record (include/msb_q4.h)."""
    return _lib.load().msb_q4_record_bytes(ctypes.byref(dims.c()))


def pack(gate: np.ndarray, up: np.ndarray, down: np.ndarray, router: np.ndarray, dims: Dims,
         threads: int = 0) -> dict:
    """Pack model-layout BF16 weights (uint16 bit arrays) with libmsb's host packer.

    gate, up: [E][I][d]; down: [E][d][I]; router: [d][E].
    Returns numpy arrays: records [E][I][3d] u16, sketch u32, alpha [E][Ipad] f32,
    router_t [E][d] u16.
    """
    lib = _lib.load()
    E, I, d = dims.experts, dims.inter, dims.d
    for a, shape in ((gate, (E, I, d)), (up, (E, I, d)), (down, (E, d, I)), (router, (d, E))):
        if a.dtype != np.uint16 or a.shape != shape or not a.flags.c_contiguous:
            raise ValueError("expected contiguous uint16 array of shape %s, got %s %s"
                             % (shape, a.dtype, a.shape))
    cd = dims.c()
    words = lib.msb_sketch_words(ctypes.byref(cd))
    if words == 0:
        _check(_lib.MSB_EINVAL, "msb_sketch_words")
    records = np.empty((E, I, 3 * d), np.uint16)
    sketch = np.empty(words, np.uint32)
    alpha = np.empty((E, dims.ipad), np.float32)
    router_t = np.empty((E, d), np.uint16)
    rc = lib.msb_pack(_ptr(gate), _ptr(up), _ptr(down), _ptr(router), ctypes.byref(cd),
                      _ptr(records), _ptr(sketch), _ptr(alpha), _ptr(router_t), threads)
    _check(rc, "msb_pack")
    return {"records": records, "sketch": sketch, "alpha": alpha, "router_t": router_t}


def pack_q4(gate: np.ndarray, up: np.ndarray, down: np.ndarray, router: np.ndarray, dims: Dims,
            threads: int = 0) -> dict:
    """Pack model-layout BF16 weights into 4-bit channel records (format in
    include/msb_q4.h) with libmsb's host packer.

    gate, up: [E][I][d]; down: [E][d][I]; router: [d][E] (uint16 BF16 bits).
    Returns numpy arrays: records [E][I][msb_q4_record_bytes] u8, sketch u32 and
    alpha [E][Ipad] f32 of the dequantised gate rows, router_t [E][d] u16.
    """
    lib = _lib.load()
    E, I, d = dims.experts, dims.inter, dims.d
    for a, shape in ((gate, (E, I, d)), (up, (E, I, d)), (down, (E, d, I)), (router, (d, E))):
        if a.dtype != np.uint16 or a.shape != shape or not a.flags.c_contiguous:
            raise ValueError("expected contiguous uint16 array of shape %s, got %s %s"
                             % (shape, a.dtype, a.shape))
    cd = dims.c()
    rb = lib.msb_q4_record_bytes(ctypes.byref(cd))
    words = lib.msb_sketch_words(ctypes.byref(cd))
    if rb == 0 or words == 0:
        _check(_lib.MSB_EINVAL, "msb_q4_record_bytes / msb_sketch_words")
    records = np.empty((E, I, rb), np.uint8)
    sketch = np.empty(words, np.uint32)
    alpha = np.empty((E, dims.ipad), np.float32)
    router_t = np.empty((E, d), np.uint16)
    rc = lib.msb_pack_q4(_ptr(gate), _ptr(up), _ptr(down), _ptr(router), ctypes.byref(cd),
                         _ptr(records), _ptr(sketch), _ptr(alpha), _ptr(router_t), threads)
    _check(rc, "msb_pack_q4")
    return {"records": records, "sketch": sketch, "alpha": alpha, "router_t": router_t}


# ------------------------------------------------------------------ device objects

class PackedLayer:
    """One MoE layer's packed weights resident on a CUDA device."""

    def __init__(self, dims: Dims, records, sketch, alpha, router_t, lr_a=None, lr_b=None, q4=False):
        """q4: records are 4-bit channel records (msb_pack_q4: uint8 [E][I][record bytes])."""
        self.dims = dims
        self.records, self.sketch, self.alpha, self.router_t = records, sketch, alpha, router_t
        self.lr_a, self.lr_b = lr_a, lr_b
        self.q4 = q4
        self._check()

    def _check(self):
        """Sizes, element types and device of every tensor against the dims, so that the
        kernels never read past a buffer (done once, at construction)."""
        d, I, E, r = self.dims.d, self.dims.inter, self.dims.experts, self.dims.rank
        words = sketch_words(self.dims)
        if words == 0:
            raise ValueError("dims rejected by the library: %s" % (self.dims,))
        rec = ((E * I * q4_record_bytes(self.dims), 1) if self.q4 else (E * I * 3 * d, 2))
        want = [("records", self.records) + rec, ("sketch", self.sketch, words, 4),
                ("alpha", self.alpha, E * self.dims.ipad, 4), ("router_t", self.router_t, E * d, 2)]
        if r > 0:
            want += [("lr_a", self.lr_a, E * d * r, 2), ("lr_b", self.lr_b, E * r * d, 2)]
        dev = self.records.device
        for name, t, numel, size in want:
            if t is None:
                raise ValueError("%s is required (rank %d)" % (name, r))
            if (t.numel() != numel or t.element_size() != size or not t.is_contiguous() or
                    t.device != dev or (name == "alpha" and not t.dtype.is_floating_point)):
                raise ValueError("%s: expected %d contiguous %d-byte elements on %s, got %s %s on %s"
                                 % (name, numel, size, dev, t.dtype, tuple(t.shape), t.device))

    @classmethod
    def from_host(cls, dims: Dims, packed: dict, lr_a: np.ndarray | None, lr_b: np.ndarray | None,
                  device="cuda"):
        """Upload host arrays (``pack`` output, BF16 factor bits).  Factors of a rank above
        dims.rank contribute their first dims.rank columns of A_e and rows of B_e."""
        import torch

        def t(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        r = dims.rank
        if r > 0 and lr_a is not None and lr_b is not None:
            # factors of a higher rank: the first r columns of A_e and rows of B_e
            lr_a, lr_b = lr_a[:, :, :r], lr_b[:, :r, :]
        q4 = packed["records"].dtype == np.uint8  # pack_q4 output
        return cls(dims, t(packed["records"] if q4 else packed["records"].view(np.int16)),
                   t(packed["sketch"].view(np.int32)), t(packed["alpha"]), t(packed["router_t"].view(np.int16)),
                   None if lr_a is None or r == 0 else t(lr_a.view(np.int16)),
                   None if lr_b is None or r == 0 else t(lr_b.view(np.int16)), q4=q4)

    def clone(self) -> "PackedLayer":
        """A copy at different addresses (same values)."""
        c = lambda a: None if a is None else a.clone()
        return PackedLayer(self.dims, c(self.records), c(self.sketch), c(self.alpha),
                           c(self.router_t), c(self.lr_a), c(self.lr_b), q4=self.q4)

    def without_lowrank(self) -> "PackedLayer":
        """The same weights (shared, not copied) with rank 0: no compensation term."""
        d = self.dims
        return PackedLayer(Dims(d.d, d.inter, d.experts, d.top_e, 0, d.renorm), self.records,
                           self.sketch, self.alpha, self.router_t, None, None, q4=self.q4)

    def nbytes(self) -> int:
        return sum(a.numel() * a.element_size() for a in
                   (self.records, self.sketch, self.alpha, self.router_t, self.lr_a, self.lr_b)
                   if a is not None)


def workspace_size(dims: Dims, max_batch: int) -> int:
    return _lib.load().msb_workspace_size(ctypes.byref(dims.c()), max_batch)


class Workspace:
    """Zero-filled device scratch for calls of up to max_batch tokens."""

    def __init__(self, dims: Dims, max_batch: int, device="cuda"):
        import torch
        n = workspace_size(dims, max_batch)
        if n == 0:
            raise ValueError("invalid dims or batch for a workspace")
        self.nbytes = n
        self.buf = torch.zeros(n + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256

    def check(self, stream=None):
        rc = _lib.load().msb_check(self.ptr, _stream(stream))
        _check(rc, "kernel")


class Trace:
    """Device buffers receiving a call's routing and selection."""

    def __init__(self, dims: Dims, batch: int, k: int, device="cuda", scores=False,
                 threshold=False, union=True):
        """union=False leaves out the per-expert union count (batches above 1 that trace it
        take the multi-kernel path)."""
        import torch
        K = dims.top_e
        cap = dims.inter if threshold else k
        self.expert_ids = torch.zeros((batch, K), dtype=torch.int32, device=device)
        self.expert_w = torch.zeros((batch, K), dtype=torch.float32, device=device)
        self.sel = torch.zeros((batch, K, cap), dtype=torch.int16, device=device)
        self.sel_count = torch.zeros((batch, K), dtype=torch.int32, device=device)
        self.union_count = (torch.zeros((dims.experts,), dtype=torch.int32, device=device)
                            if union else None)
        self.scores = (torch.zeros((batch, K, dims.ipad), dtype=torch.float32, device=device)
                       if scores else None)

    def c(self) -> MsbTrace:
        return MsbTrace(_ptr(self.expert_ids), _ptr(self.expert_w), _ptr(self.sel),
                        _ptr(self.sel_count), _ptr(self.union_count), _ptr(self.scores))


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _temporaries_on(stream, tensors):
    """Buffers a call allocates for the caller (out, workspace) come from torch's current
    stream.  When the call runs on another stream, order that stream after their
    allocation and zero-fill, and tell the caching allocator that the stream uses them.
    A raw stream handle cannot be ordered from here: the caller passes the buffers."""
    tensors = [t for t in tensors if t is not None]
    if stream is None or not tensors:
        return
    if isinstance(stream, int):
        raise ValueError("with a raw stream handle, pass out= and workspace= allocated for it")
    import torch
    cur = torch.cuda.current_stream(stream.device)
    if stream != cur:
        stream.wait_stream(cur)
        for t in tensors:
            t.record_stream(stream)


def _check_call(x, layer: PackedLayer, out, trace, K: int, cap: int):
    """Checks the C ABI cannot make (it sees raw pointers), done before anything is
    allocated or launched: x on the current device; layer, out and trace on x's device;
    out shaped like x; the
    trace laid out for this call (K routed experts per token, `cap` channels per
    (token, expert) in sel, at least x's batch of rows)."""
    dev = x.device
    if dev.type == "cuda":
        import torch
        if dev.index != torch.cuda.current_device():
            raise ValueError("x is on %s but the current device is cuda:%d (the library "
                             "launches on the current device)" % (dev, torch.cuda.current_device()))
    if layer.records.device != dev:
        raise ValueError("the layer is on %s, x on %s" % (layer.records.device, dev))
    if out is not None and (out.shape != x.shape or out.dtype != x.dtype or
                            not out.is_contiguous() or out.device != dev):
        raise ValueError("out must be a contiguous bf16 tensor shaped like x, on x's device")
    if trace is None:
        return
    B, dims = x.shape[0], layer.dims
    want = {"expert_ids": (K,), "expert_w": (K,), "sel_count": (K,), "sel": (K, cap)}
    if trace.scores is not None:
        want["scores"] = (K, dims.ipad)
    for name, tail in want.items():
        t = getattr(trace, name)
        if (t.dim() != 1 + len(tail) or t.shape[0] < B or tuple(t.shape[1:]) != tail or
                not t.is_contiguous() or t.device != dev):
            raise ValueError("trace.%s is %s on %s; this call needs [>= %d]%s on %s"
                             % (name, tuple(t.shape), t.device, B, list(tail), dev))
    u = trace.union_count
    if u is not None and (u.dim() != 1 or u.shape[0] < dims.experts or u.device != dev):
        raise ValueError("trace.union_count needs >= %d entries on %s" % (dims.experts, dev))


def _act(x, dims: Dims):
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != dims.d or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 [batch][d] tensor")
    return x


# ------------------------------------------------------------------ the block

def moe_sparse_block(x, layer: PackedLayer, k: int, out=None, workspace: Workspace | None = None,
                     trace: Trace | None = None, general: bool = False, stream=None,
                     top_e: int | None = None, single: bool = False):
    """One sparse-MoE block decode step: out[t] = sum_e w_te * (gathered SwiGLU over the
    k top-scoring channels + A_e B_e x_t).  x: bf16 [B][d] on the GPU.  top_e: route each
    token to this many experts instead of the trained layer.dims.top_e (at most that).
    general / single: the multi-kernel path at any batch / the single-launch kernel up to
    16 tokens (default: whichever the measured crossover for d prefers; see path_info).
    out and workspace are allocated when not given (pass both for repeated calls and for
    a raw stream handle); the call is asynchronous on `stream` (default: torch's current
    stream)."""
    import torch
    dims = layer.dims
    _act(x, dims)
    _check_call(x, layer, out, trace, dims.top_e if top_e is None else top_e, k)
    B = x.shape[0]
    new_out = new_ws = None
    if out is None:
        out = new_out = torch.empty_like(x)
    if workspace is None:
        workspace = new_ws = Workspace(dims, B, x.device)
    _temporaries_on(stream, [new_out, new_ws.buf if new_ws else None])
    tr = trace.c() if trace is not None else None
    flags = (_lib.MSB_FLAG_GENERAL if general else 0) | (_lib.MSB_FLAG_SINGLE if single else 0)
    args = (_ptr(x), B, _ptr(layer.router_t), _ptr(layer.records), _ptr(layer.sketch),
            _ptr(layer.alpha), k)
    rest = (_ptr(layer.lr_a), _ptr(layer.lr_b), _ptr(out), ctypes.byref(dims.c()), workspace.ptr,
            workspace.nbytes, ctypes.byref(tr) if tr is not None else None, flags, _stream(stream))
    if layer.q4:
        if top_e is not None:
            raise ValueError("4-bit records: the expert-count override is not available")
        rc = _lib.load().moe_sparse_block_q4(*args, *rest)
    elif top_e is None:
        rc = _lib.load().moe_sparse_block(*args, *rest)
    else:
        rc = _lib.load().moe_sparse_block_top_e(*args, top_e, *rest)
    _check(rc, "moe_sparse_block")
    return out


def noalloc_check(stream=None):
    """Raise MsbError if the last moe_sparse_block_noalloc call on the current device
    was flagged by its kernel (synchronises the stream; clears the flag)."""
    _check(_lib.load().msb_noalloc_check(_stream(stream)), "moe_sparse_block_noalloc kernel")


def moe_sparse_block_noalloc(x, layer: PackedLayer, k: int, out=None, trace: Trace | None = None,
                             stream=None):
    """The batch-1 block without a workspace (scratch is a static device array of
    the library), for callers that cannot allocate device memory.  Read the call's
    kernel status with noalloc_check() before the next such call."""
    if layer.q4:
        raise ValueError("4-bit records: use moe_sparse_block")
    import torch
    dims = layer.dims
    _act(x, dims)
    if x.shape[0] != 1:
        raise ValueError("moe_sparse_block_noalloc takes one token")
    _check_call(x, layer, out, trace, dims.top_e, k)
    if out is None:
        out = torch.empty_like(x)
        _temporaries_on(stream, [out])
    tr = trace.c() if trace is not None else None
    rc = _lib.load().moe_sparse_block_noalloc(
        _ptr(x), _ptr(layer.router_t), _ptr(layer.records), _ptr(layer.sketch), _ptr(layer.alpha),
        k, _ptr(layer.lr_a), _ptr(layer.lr_b), _ptr(out), ctypes.byref(dims.c()),
        ctypes.byref(tr) if tr is not None else None, _stream(stream))
    _check(rc, "moe_sparse_block_noalloc")
    return out


class HostCall:
    """Repeated block calls on activations in host memory (moe_sparse_block_host): each
    call copies one [batch][d] bf16 host tensor to the device, runs the block and copies
    the result back into a host tensor, all enqueued on `stream`.

    The layer, k, batch, device staging buffers, workspace and stream are fixed and
    checked once, here; a call passes only the two host buffers (pinned host tensors of
    shape [batch][d], bf16), so the per-step cost on the host is one C call.  The call is
    asynchronous: synchronise the stream before reading `out_host` or reusing `x_host`.

    x_ready=True declares that nothing earlier on the stream writes x_host (the host
    produced it before the call), so that the single-launch kernel fetches it while the
    previous launch still runs (MSB_FLAG_X_READY).  general / single: as for
    moe_sparse_block."""

    def __init__(self, layer: PackedLayer, k: int, batch: int, stream=None, general: bool = False,
                 x_ready: bool = False, single: bool = False):
        if layer.q4:
            raise ValueError("4-bit records: use moe_sparse_block")
        import torch
        dims = layer.dims
        if not 1 <= k <= dims.inter:
            raise ValueError("k must lie in 1..%d" % dims.inter)
        dev = layer.records.device
        self.batch, self.d = batch, dims.d
        self.x_dev = torch.empty((batch, dims.d), dtype=torch.bfloat16, device=dev)
        self.out_dev = torch.empty_like(self.x_dev)
        self.workspace = Workspace(dims, batch, dev)
        self._dims = dims.c()
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        _temporaries_on(self.stream, [self.x_dev, self.out_dev, self.workspace.buf])
        self._fn = _lib.load().moe_sparse_block_host
        self._head = (_ptr(self.x_dev), batch, _ptr(layer.router_t), _ptr(layer.records),
                      _ptr(layer.sketch), _ptr(layer.alpha), k, _ptr(layer.lr_a), _ptr(layer.lr_b),
                      _ptr(self.out_dev))
        flags = ((_lib.MSB_FLAG_GENERAL if general else 0) | (_lib.MSB_FLAG_X_READY if x_ready else 0)
                 | (_lib.MSB_FLAG_SINGLE if single else 0))
        self._tail = (ctypes.byref(self._dims), self.workspace.ptr, self.workspace.nbytes, flags,
                      _stream(self.stream))
        self._layer = layer  # keep the weights alive

    def check_host(self, t):
        """A host tensor this call can take (shape, dtype, pinned, contiguous)."""
        import torch
        if (t.device.type != "cpu" or t.dtype != torch.bfloat16 or tuple(t.shape) != (self.batch, self.d)
                or not t.is_contiguous() or not t.is_pinned()):
            raise ValueError("expected a pinned contiguous bf16 host tensor of shape [%d][%d]"
                             % (self.batch, self.d))
        return t

    def __call__(self, x_host, out_host):
        """x_host, out_host: host tensors accepted by check_host, or their data pointers."""
        xp = x_host if isinstance(x_host, int) else x_host.data_ptr()
        op = out_host if isinstance(out_host, int) else out_host.data_ptr()
        rc = self._fn(xp, *self._head, op, *self._tail)
        if rc != _lib.MSB_OK:
            raise MsbError(rc, "moe_sparse_block_host")


def moe_sparse_block_threshold(x, layer: PackedLayer, tau: float, out=None,
                               workspace: Workspace | None = None, trace: Trace | None = None,
                               stream=None):
    """The calibrated-threshold comparator: channels with score > tau."""
    if layer.q4:
        raise ValueError("4-bit records: use moe_sparse_block")
    import torch
    dims = layer.dims
    _act(x, dims)
    _check_call(x, layer, out, trace, dims.top_e, dims.inter)
    B = x.shape[0]
    new_out = new_ws = None
    if out is None:
        out = new_out = torch.empty_like(x)
    if workspace is None:
        workspace = new_ws = Workspace(dims, B, x.device)
    _temporaries_on(stream, [new_out, new_ws.buf if new_ws else None])
    tr = trace.c() if trace is not None else None
    rc = _lib.load().moe_sparse_block_threshold(
        _ptr(x), B, _ptr(layer.router_t), _ptr(layer.records), _ptr(layer.sketch),
        _ptr(layer.alpha), float(tau), _ptr(layer.lr_a), _ptr(layer.lr_b), _ptr(out),
        ctypes.byref(dims.c()), workspace.ptr, workspace.nbytes,
        ctypes.byref(tr) if tr is not None else None, _stream(stream))
    _check(rc, "moe_sparse_block_threshold")
    return out


def path_info(dims: Dims, batch: int, k: int, general: bool = False, single: bool = False) -> dict:
    """Which path moe_sparse_block takes on the current device, and its plan."""
    info = (ctypes.c_int32 * 8)()
    flags = (_lib.MSB_FLAG_GENERAL if general else 0) | (_lib.MSB_FLAG_SINGLE if single else 0)
    rc = _lib.load().msb_path_info(ctypes.byref(dims.c()), batch, k, flags, info)
    _check(rc, "msb_path_info")
    v = list(info)
    return {"path": "single_launch" if v[0] == 1 else "multi_kernel", "cluster_size": v[1],
            "clusters_per_expert": v[2], "ring_slots": v[3], "smem_bytes": v[4],
            "resident_clusters16": v[5], "resident_clusters8": v[6]}


def residual_rmsnorm(h, y, x_next, eps: float = 1e-6, stream=None):
    """h += y (FP32 residual, y bf16 or None); x_next = BF16(RMSNorm(h))."""
    import torch
    if h.dtype != torch.float32 or h.dim() != 2 or not h.is_contiguous():
        raise ValueError("h must be a contiguous float32 [batch][d] tensor")
    for name, t in (("y", y), ("x_next", x_next)):
        if t is not None and (t.shape != h.shape or t.dtype != torch.bfloat16 or
                              not t.is_contiguous() or t.device != h.device):
            raise ValueError("%s must be a contiguous bf16 tensor shaped like h, on h's device" % name)
    B, d = h.shape
    rc = _lib.load().msb_residual_rmsnorm(_ptr(h), _ptr(y), _ptr(x_next), B, d, float(eps),
                                          _stream(stream))
    _check(rc, "msb_residual_rmsnorm")
    return x_next


def calibrate_threshold(scores: np.ndarray, budget: float) -> float:
    """Offline calibration of the threshold comparator (not part of the decode path).

    The reading of "The threshold promises a budget but does not keep it": tau is the
    pooled calibration score with exactly m = floor(N * budget) scores above it when
    there are no ties, i.e. the (m+1)-th largest.  Found here by linear-time selection
    (the element of ascending rank N - 1 - m), not by a full sort."""
    s = np.asarray(scores, dtype=np.float64).ravel()
    if s.size == 0:
        raise ValueError("no calibration scores")
    m = min(int(np.floor(s.size * budget)), s.size - 1)
    r = s.size - 1 - m
    return float(np.partition(s, r)[r])
