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


def header_functions():
    text = open(os.path.join(ROOT, "include", "msb.h")).read()
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
