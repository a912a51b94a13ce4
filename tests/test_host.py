"""CPU tests of the host side of libmsb: exports, the packer, argument checks.

No GPU is touched: the packer is host code and every argument check returns
before anything is enqueued.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def msb():
    from token_top_expert_b200 import build
    build.build()
    import token_top_expert_b200 as m
    m.load_library()
    return m


INSTR_HEADER = "msb_instr.h"  # entry points of the instrumented build only


def header_functions(instrumented=False):
    inc = os.path.join(ROOT, "include")
    names = [f for f in sorted(os.listdir(inc)) if f.endswith(".h")]
    names = [f for f in names if (f == INSTR_HEADER) == instrumented]
    text = "".join(open(os.path.join(inc, f)).read() for f in names)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(msb):
    from token_top_expert_b200 import _lib
    declared = header_functions()
    assert len(declared) >= 10
    assert sorted(_lib.SYMBOLS) == declared
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    # the product library carries none of the instrumented build's entry points
    for name in header_functions(instrumented=True):
        assert not hasattr(lib, name), name


def test_instrumented_library_exports_its_entry_points():
    from token_top_expert_b200 import build
    path = build.build(variant="instr")
    lib = ctypes.CDLL(path)
    extra = header_functions(instrumented=True)
    assert extra == ["msb_debug_inject", "msb_debug_set_marks"]
    for name in header_functions() + extra:
        assert hasattr(lib, name), name
    lib.msb_debug_inject.restype = ctypes.c_int32
    lib.msb_debug_inject.argtypes = [ctypes.c_uint32, ctypes.c_uint64]
    assert lib.msb_debug_inject(3, 0) == -1   # MSB_EINVAL: no such injection
    assert lib.msb_debug_inject(0, 0) == 0


def decode_sketch(words, dims, e):
    """Reference decoder of the packed sketch format documented in include/msb.h:
    [tile][chunk][lane][h] words; pair q of a word covers columns
    64*chunk + 16*(q//2) + 2*(lane%4) + 8*(q%2) (+1) of row 16*tile + lane//4 + 8*h,
    2-bit codes (sign, magnitude) at bits (15-2q, 14-2q) and (31-2q, 30-2q)."""
    d, ipad = dims.d, dims.ipad
    KC, nt = d // 64, ipad // 16
    t = np.zeros((ipad, d), np.int8)
    base = e * nt * KC * 64
    for rt in range(nt):
        for kc in range(KC):
            blk = words[base + (rt * KC + kc) * 64: base + (rt * KC + kc + 1) * 64]
            for lane in range(32):
                g, c = lane >> 2, lane & 3
                for h in range(2):
                    w = int(blk[lane * 2 + h])
                    row = rt * 16 + g + 8 * h
                    for q in range(8):
                        col = kc * 64 + 16 * (q >> 1) + 2 * c + 8 * (q & 1)
                        for off, sh in ((0, 14 - 2 * q), (1, 30 - 2 * q)):
                            code = (w >> sh) & 3
                            assert code != 2, "invalid code (sign without magnitude)"
                            t[row, col + off] = {0: 0, 1: 1, 3: -1}[code]
    return t


@pytest.mark.parametrize("d,inter", [(256, 512), (256, 33), (64, 33), (192, 48)])
def test_packer_matches_oracle_sketch(msb, d, inter):
    w = synth.TINY.with_(d=d, inter=inter, experts=3, heavy_frac=0.05, heavy_scale=4.0)
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, w.rank)
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    for e in range(w.experts):
        t_ref, a_ref = oracle.ternary_sketch(oracle.bf16_to_f64(lw.gate[e]))
        t = decode_sketch(pk["sketch"], dims, e)
        np.testing.assert_array_equal(t[:inter], t_ref)
        assert not t[inter:].any()
        np.testing.assert_array_equal(pk["alpha"][e, :inter], a_ref)
        assert not pk["alpha"][e, inter:].any()
        # records: gate row | up row | down column
        np.testing.assert_array_equal(pk["records"][e, :, :w.d], lw.gate[e])
        np.testing.assert_array_equal(pk["records"][e, :, w.d:2 * w.d], lw.up[e])
        np.testing.assert_array_equal(pk["records"][e, :, 2 * w.d:], lw.down[e].T)
    np.testing.assert_array_equal(pk["router_t"], lw.router.T)


def test_packer_exact_threshold_tie(msb):
    # d = 64, row = [7, 512, 64, 32, 16, 8, 1, 0, ...] * 2**-10: sum = 640 * 2**-10,
    # delta = 0.7 * sum / 64 = 7 * 2**-10 = the first entry, which must NOT be kept.
    d, I = 64, 16
    dims = msb.Dims(d, I, 1, 1, 0)
    row = np.zeros(d, np.float32)
    row[:7] = np.array([7, 512, 64, 32, 16, 8, 1], np.float32) * 2.0 ** -10
    row[3] = -row[3]
    gate = np.zeros((1, I, d), np.uint16)
    gate[0, 0] = synth.f32_to_bf16_bits(row)
    t_ref, a_ref = oracle.ternary_sketch(oracle.bf16_to_f64(gate[0]))
    assert list(t_ref[0, :8]) == [0, 1, 1, -1, 1, 1, 0, 0]
    assert a_ref[0] == np.float32(632 / 5 * 2.0 ** -10)
    pk = msb.pack(gate, gate.copy(), np.zeros((1, d, I), np.uint16), np.zeros((d, 1), np.uint16),
                  dims)
    t = decode_sketch(pk["sketch"], dims, 0)
    np.testing.assert_array_equal(t[:I], t_ref)
    np.testing.assert_array_equal(pk["alpha"][0, :I], a_ref)


def decode_q4_records(rec, d):
    """Reference decoder of the 4-bit record format documented in include/msb_q4.h:
    3d nibble codes (element 2i in bits 0-3 of byte i, element 2i+1 in bits 4-7), then
    (scale, bias) BF16 pairs of the gate row's, the up row's and the down column's
    groups of 64, then zero padding.  rec: [n][record bytes] u8.
    Returns q [n][3][d], s [n][3][d/64], b [n][3][d/64] (float64), padding bytes."""
    n, g = rec.shape[0], d // 64
    nib = rec[:, :3 * d // 2]
    q = np.empty((n, 3 * d), np.uint8)
    q[:, 0::2] = nib & 0xF
    q[:, 1::2] = nib >> 4
    par = np.ascontiguousarray(rec[:, 3 * d // 2: 3 * d // 2 + 12 * g]).view(np.uint16)
    par = par.reshape(n, 3, g, 2)
    return (q.reshape(n, 3, d), oracle.bf16_to_f64(par[..., 0]), oracle.bf16_to_f64(par[..., 1]),
            rec[:, 3 * d // 2 + 12 * g:])


@pytest.mark.parametrize("d,inter", [(256, 40), (64, 33), (192, 17)])
def test_q4_packer_matches_oracle(msb, d, inter):
    """4-bit records, sketch and alpha against the oracle's quantiser (oracle.q4) and
    its sketch of the dequantised gate rows, bit for bit; includes a zero gate row, a
    constant group and heavy rows."""
    w = synth.TINY.with_(d=d, inter=inter, experts=2, heavy_frac=0.1, heavy_scale=4.0)
    lw = synth.layer_weights(w)
    gate, up, down = lw.gate.copy(), lw.up.copy(), lw.down.copy()
    gate[0, 1] = 0
    up[1, 2, :64] = synth.f32_to_bf16_bits(np.full(64, -0.375, np.float32))
    dims = msb.Dims(d, inter, w.experts, w.top_e, 0)
    pk = msb.pack_q4(gate, up, down, lw.router, dims)
    rb = oracle.q4.record_bytes(d)
    assert pk["records"].shape == (w.experts, inter, rb)
    for e in range(w.experts):
        q, s, b, pad = decode_q4_records(pk["records"][e], d)
        assert not pad.any()
        for part, mat in enumerate((gate[e], up[e], down[e].T)):
            q_ref, s_ref, b_ref = oracle.q4.quantize_groups(oracle.bf16_to_f64(mat))
            np.testing.assert_array_equal(q[:, part], q_ref)
            np.testing.assert_array_equal(s[:, part], s_ref)
            np.testing.assert_array_equal(b[:, part], b_ref)
        g_deq = oracle.q4.q4_weights(oracle.bf16_to_f64(gate[e]), oracle.bf16_to_f64(up[e]),
                                     oracle.bf16_to_f64(down[e]))[0]
        t_ref, a_ref = oracle.ternary_sketch(g_deq)
        np.testing.assert_array_equal(decode_sketch(pk["sketch"], dims, e)[:inter], t_ref)
        np.testing.assert_array_equal(pk["alpha"][e, :inter], a_ref)
    np.testing.assert_array_equal(pk["router_t"], lw.router.T)


def test_q4_argument_checks(msb):
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    for d, want in ((2048, 3456), (64, 112), (96, 0), (0, 0), (16384, 0)):
        assert lib.msb_q4_record_bytes(ctypes.byref(msb.Dims(d, 8, 1, 1, 0).c())) == want
    assert lib.msb_q4_record_bytes(None) == 0
    z = np.zeros(64 * 8, np.uint16)
    out = np.zeros(1 << 16, np.uint8)
    for dims, want in ((msb.Dims(96, 8, 1, 1, 0), _lib.MSB_EINVAL),
                       (msb.Dims(64, 0, 1, 1, 0), _lib.MSB_EINVAL),
                       (msb.Dims(64, _lib.MSB_MAX_INTER + 1, 1, 1, 0), _lib.MSB_EUNSUPPORTED)):
        rc = lib.msb_pack_q4(z.ctypes.data, z.ctypes.data, z.ctypes.data, z.ctypes.data,
                             ctypes.byref(dims.c()), out.ctypes.data, out.ctypes.data,
                             out.ctypes.data, out.ctypes.data, 1)
        assert rc == want
    # dims the size queries reject (more routed experts than experts) are rejected by
    # both packers before anything is written, and by the bindings before allocating
    bad = msb.Dims(64, 8, 2, 3, 0)
    assert lib.msb_sketch_words(ctypes.byref(bad.c())) == 0
    for fn in (lib.msb_pack, lib.msb_pack_q4):
        rc = fn(z.ctypes.data, z.ctypes.data, z.ctypes.data, z.ctypes.data, ctypes.byref(bad.c()),
                out.ctypes.data, out.ctypes.data, out.ctypes.data, out.ctypes.data, 1)
        assert rc == _lib.MSB_EINVAL
    g = np.zeros((2, 8, 64), np.uint16)
    for fn in (msb.pack, msb.pack_q4):
        with pytest.raises(msb.MsbError):
            fn(g, g, np.zeros((2, 64, 8), np.uint16), np.zeros((64, 2), np.uint16), bad)
    rc = lib.msb_pack_q4(None, z.ctypes.data, z.ctypes.data, z.ctypes.data,
                         ctypes.byref(msb.Dims(64, 8, 1, 1, 0).c()), out.ctypes.data,
                         out.ctypes.data, out.ctypes.data, out.ctypes.data, 1)
    assert rc == _lib.MSB_EINVAL


def test_argument_checks_without_gpu(msb):
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    dims = _lib.MsbDims(2048, 768, 128, 8, 32, 1)
    ws = lib.msb_workspace_size(ctypes.byref(dims), 1)
    assert ws > 0
    assert lib.msb_workspace_size(ctypes.byref(dims), 0) == 0
    assert lib.msb_workspace_size(ctypes.byref(dims), 257) == 0
    assert lib.msb_sketch_words(ctypes.byref(dims)) == 128 * 768 * 2048 // 16
    fake = 1 << 20  # never dereferenced: every call below fails its checks first

    def call(x=fake, batch=1, k=138, out=fake * 2, d=dims, ws_bytes=ws, rt=fake, wsp=fake,
             lr=fake):
        return lib.moe_sparse_block(x, batch, rt, fake, fake, fake, k, lr, lr, out,
                                    ctypes.byref(d), wsp, ws_bytes, None, 0, None)

    assert call(x=None) == _lib.MSB_EINVAL
    assert call(k=0) == _lib.MSB_EINVAL
    assert call(k=769) == _lib.MSB_EINVAL
    assert call(batch=0) == _lib.MSB_EINVAL
    assert call(batch=257) == _lib.MSB_EUNSUPPORTED
    assert call(ws_bytes=ws - 1) == _lib.MSB_EINVAL
    assert call(x=fake + 8) == _lib.MSB_EINVAL          # misaligned
    assert call(out=fake + 1024) == _lib.MSB_EINVAL     # out overlaps x
    assert call(lr=None) == _lib.MSB_EINVAL             # rank 32 needs A, B
    bad = _lib.MsbDims(2000, 768, 128, 8, 32, 1)        # d % 64 != 0
    assert call(d=bad) == _lib.MSB_EINVAL
    bad = _lib.MsbDims(2048, 768, 128, 129, 32, 1)      # top_e > E
    assert call(d=bad) == _lib.MSB_EINVAL
    bad = _lib.MsbDims(2048, 8192, 128, 8, 32, 1)       # I beyond the compiled limit
    assert call(d=bad) == _lib.MSB_EUNSUPPORTED
    # expert-count override: at most the trained top_e, at least 1
    def call_top_e(top_e, x=fake):
        return lib.moe_sparse_block_top_e(x, 1, fake, fake, fake, fake, 138, top_e, fake, fake,
                                          fake * 2, ctypes.byref(dims), fake, ws, None, 0, None)

    assert call_top_e(9) == _lib.MSB_EINVAL
    assert call_top_e(0) == _lib.MSB_EINVAL
    assert call_top_e(4, x=None) == _lib.MSB_EINVAL
    assert lib.msb_residual_rmsnorm(None, None, fake, 1, 2048, 1e-6, None) == _lib.MSB_EINVAL
    assert lib.msb_strerror(_lib.MSB_ETIMEOUT) == b"a kernel's bounded wait ran out"


def test_raw_stream_handle_needs_caller_buffers():
    """Buffers the binding allocates live on torch's current stream; with a raw handle
    it cannot order them, so it refuses instead of racing (checked before any CUDA call)."""
    from token_top_expert_b200 import block
    block._temporaries_on(None, [object()])       # default stream: nothing to order
    block._temporaries_on(12345, [None, None])    # caller gave every buffer
    with pytest.raises(ValueError):
        block._temporaries_on(12345, [object()])


def test_binding_checks_buffers_before_launch(msb):
    """The binding refuses buffers the kernels would overrun or misread -- out not
    shaped like x, a trace laid out for another K or k, tensors on another device --
    before it allocates or launches anything (CPU tensors stand in for device ones;
    every case raises before the C call)."""
    import torch
    dims = msb.Dims(64, 40, 4, 2, 0)
    z = lambda *s, dt=torch.int16, dev="cpu": torch.zeros(*s, dtype=dt, device=dev)  # noqa: E731
    words = msb.sketch_words(dims)

    def fake_layer(dev="cpu"):
        return msb.PackedLayer(dims, z(4, 40, 3 * 64, dev=dev), z(words, dt=torch.int32, dev=dev),
                               z(4, 48, dt=torch.float32, dev=dev), z(4, 64, dev=dev))

    layer = fake_layer()
    x = z(3, 64, dt=torch.bfloat16)
    with pytest.raises(ValueError, match="out"):
        msb.moe_sparse_block(x, layer, 8, out=z(2, 64, dt=torch.bfloat16))
    with pytest.raises(ValueError, match="out"):
        msb.moe_sparse_block(x, layer, 8, out=z(3, 64))                       # int16, not bf16
    with pytest.raises(ValueError, match="out"):
        msb.moe_sparse_block(x, layer, 8, out=z(64, 3, dt=torch.bfloat16).t())
    with pytest.raises(ValueError, match="trace.sel "):
        msb.moe_sparse_block(x, layer, 8, trace=msb.Trace(dims, 3, 9, device="cpu"))
    with pytest.raises(ValueError, match="trace.expert_ids"):
        msb.moe_sparse_block(x, layer, 8, trace=msb.Trace(dims, 2, 8, device="cpu"))  # 2 < 3 rows
    with pytest.raises(ValueError, match="trace.expert_ids"):
        msb.moe_sparse_block(x, layer, 8, top_e=1, trace=msb.Trace(dims, 3, 8, device="cpu"))
    with pytest.raises(ValueError, match="trace.sel "):                      # needs capacity I
        msb.moe_sparse_block_threshold(x, layer, 0.5, trace=msb.Trace(dims, 3, 8, device="cpu"))
    with pytest.raises(ValueError, match="trace.scores"):
        tr = msb.Trace(dims, 3, 8, device="cpu")
        tr.scores = z(3, 2, 40, dt=torch.float32)                            # I, not Ipad = 48
        msb.moe_sparse_block(x, layer, 8, trace=tr)
    meta = fake_layer("meta")
    with pytest.raises(ValueError, match="layer"):
        msb.moe_sparse_block(x, meta, 8)
    with pytest.raises(ValueError, match="layer"):
        msb.moe_sparse_block_noalloc(x[:1], meta, 8)
    h = z(3, 64, dt=torch.float32)
    with pytest.raises(ValueError, match="h must"):
        msb.residual_rmsnorm(h.double(), None, x)
    with pytest.raises(ValueError, match="x_next"):
        msb.residual_rmsnorm(h, None, z(3, 32, dt=torch.bfloat16))
    with pytest.raises(ValueError, match="y must"):
        msb.residual_rmsnorm(h, z(3, 64, dt=torch.float32), x)


def test_packed_layer_checks_its_tensors(msb):
    import torch
    dims = msb.Dims(64, 40, 4, 2, 2)
    z = lambda *s, dt=torch.int16: torch.zeros(*s, dtype=dt)  # noqa: E731
    ok = dict(records=z(4, 40, 192), sketch=z(msb.sketch_words(dims), dt=torch.int32),
              alpha=z(4, 48, dt=torch.float32), router_t=z(4, 64), lr_a=z(4, 64, 2), lr_b=z(4, 2, 64))
    msb.PackedLayer(dims, **ok)
    for name, bad in (("records", z(4, 40, 191)), ("sketch", z(7, dt=torch.int32)),
                      ("alpha", z(4, 40, dt=torch.float32)), ("alpha", z(4, 48, dt=torch.int32)),
                      ("router_t", z(64, 4).t()), ("lr_a", None), ("lr_b", z(4, 2, 64, dt=torch.int32))):
        with pytest.raises(ValueError, match=name):
            msb.PackedLayer(dims, **dict(ok, **{name: bad}))
    with pytest.raises(ValueError, match="dims"):
        msb.PackedLayer(msb.Dims(64, 40, 4, 5, 0), **dict(ok, lr_a=None, lr_b=None))


def test_from_host_takes_the_leading_factors_of_a_lower_rank(msb):
    dims = msb.Dims(64, 40, 4, 2, 2)
    rng = np.random.default_rng(1)
    packed = {"records": np.zeros((4, 40, 192), np.uint16),
              "sketch": np.zeros(msb.sketch_words(dims), np.uint32),
              "alpha": np.zeros((4, 48), np.float32), "router_t": np.zeros((4, 64), np.uint16)}
    a = rng.integers(0, 2**15, (4, 64, 5)).astype(np.uint16)
    b = rng.integers(0, 2**15, (4, 5, 64)).astype(np.uint16)
    lay = msb.PackedLayer.from_host(dims, packed, a, b, device="cpu")
    np.testing.assert_array_equal(lay.lr_a.numpy().view(np.uint16), a[:, :, :2])
    np.testing.assert_array_equal(lay.lr_b.numpy().view(np.uint16), b[:, :2, :])
    with pytest.raises(ValueError, match="lr_a"):
        msb.PackedLayer.from_host(msb.Dims(64, 40, 4, 2, 8), packed, a, b, device="cpu")
