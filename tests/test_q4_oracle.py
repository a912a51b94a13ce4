"""Pins of the oracle's 4-bit channel records (``oracle.q4``), CPU only.

The page that brings in 4-bit weights ("MoE top_k override (--moe-top-k)",
"Combinaison avec d'autres optimisations") does not give their format; the reading
(group-wise affine 4-bit, BF16 scale and bias per 64 weights) is stated in
``oracle/q4.py``.  The quantiser is pinned here by hand-worked groups, the rounding rule
(ties to even), the error bound s/2 that the rule implies for BF16 inputs, brute force
over the 16 codes, exact reproduction of weights that already lie on a 4-bit grid, and
the degenerate constant group; the layer wrapper by a layer whose down columns lie on a
grid along d only (a wrapper that grouped down along I would change them).
"""
import numpy as np

import oracle
import synth
from oracle import q4


def _bf16(v):
    return oracle.round_to_bf16(np.asarray(v, dtype=np.float64))


def test_hand_group():
    # w = (-1, 0.5, 2, 0.3): b = -1, s = bf16(3 / 15) = bf16(0.2) = 0.2001953125
    # (the BF16 neighbours of 0.2 are 0.19921875 and 0.2001953125); codes
    # (w + 1) / s = 0, 7.4927, 14.985, 6.4937 -> 0, 7, 15, 6.
    q, s, b = q4.quantize_groups([[-1.0, 0.5, 2.0, 0.3]], group=4)
    assert s[0, 0] == 0.2001953125 and b[0, 0] == -1.0
    assert q.tolist() == [[0, 7, 15, 6]]
    w = q4.dequantize_groups(q, s, b, group=4)
    np.testing.assert_array_equal(w, [[-1.0, 0.4013671875, 2.0029296875, 0.201171875]])


def test_codes_round_half_to_even():
    # lo = 0, hi = 15 -> s = 1, b = 0; (w - b) / s = 1.5 and 2.5 both round to 2
    q, s, b = q4.quantize_groups([[0.0, 1.5, 15.0, 2.5]], group=4)
    assert s[0, 0] == 1.0 and b[0, 0] == 0.0
    assert q.tolist() == [[0, 2, 15, 2]]


def test_constant_and_zero_groups():
    w = np.concatenate([np.full(64, 0.0), np.full(64, -0.375), np.full(64, 3.0)])[None]
    q, s, b = q4.quantize_groups(w)
    assert not q.any() and not s.any()
    np.testing.assert_array_equal(b[0], [0.0, -0.375, 3.0])
    np.testing.assert_array_equal(q4.dequantize_groups(q, s, b), w)


def _random_rows(seed, n=64, d=512):
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.02, (n, d))
    w[::7] *= 4.0                       # heavy rows, as in the synthetic workloads
    w[3, 64:128] = rng.normal(5.0, 0.05, 64)   # a narrow group far from zero: few BF16 values
    return _bf16(w)


def test_error_bound_and_extreme_codes():
    w = _random_rows(1)
    q, s, b = q4.quantize_groups(w)
    deq = q4.dequantize_groups(q, s, b)
    g = w.reshape(w.shape[0], -1, 64)
    err = np.abs(w - deq).reshape(g.shape)
    # b = min w exactly (BF16 input), so (w - b) / s lies in [0, 15 (1 + 2^-8)]: every
    # code is the nearest one and the error is at most half a step
    assert np.all(err <= s[..., None] / 2 * (1 + 1e-12))
    qg = q.reshape(g.shape)
    lo = np.take_along_axis(qg, g.argmin(-1)[..., None], -1)
    hi = np.take_along_axis(qg, g.argmax(-1)[..., None], -1)
    assert np.all(lo == 0) and np.all(hi[s > 0] == 15)


def test_codes_are_the_nearest_of_all_sixteen():
    w = _random_rows(2, n=16, d=256)
    q, s, b = q4.quantize_groups(w)
    g = w.reshape(16, -1, 64)
    codes = np.arange(16, dtype=np.float64)
    cand = s[..., None, None] * codes + b[..., None, None]        # [16][G][1][16]
    dist = np.abs(g[..., None] - cand)                              # [16][G][64][16]
    chosen = np.take_along_axis(dist, q.reshape(g.shape)[..., None].astype(np.int64), -1)[..., 0]
    np.testing.assert_array_equal(chosen, dist.min(-1))


def _grid_group(rng, exp):
    """64 weights on a 4-bit grid with BF16 scale and bias, codes 0 and 15 present."""
    s = float(_bf16(rng.uniform(1.0, 2.0) * 2.0 ** exp))
    b = float(_bf16(-rng.uniform(4.0, 10.0) * s))
    c = rng.integers(0, 16, 64)
    c[rng.integers(0, 64)] = 0
    c[(c == 0).argmax() ^ 1] = 15
    return s * c + b, c, s, b


def test_grid_weights_are_reproduced_exactly():
    rng = np.random.default_rng(3)
    groups = [_grid_group(rng, e) for e in range(-12, -2)]
    w = np.concatenate([g[0] for g in groups])[None]
    q, s, b = q4.quantize_groups(w)
    np.testing.assert_array_equal(q[0], np.concatenate([g[1] for g in groups]))
    np.testing.assert_array_equal(s[0], [g[2] for g in groups])
    np.testing.assert_array_equal(b[0], [g[3] for g in groups])
    np.testing.assert_array_equal(q4.dequantize_groups(q, s, b), w)


def test_layer_groups_down_columns_along_d():
    """Down columns on a 4-bit grid along d (a different scale per column), gate and up
    rows on a grid along d: the 4-bit layer must serve them unchanged, so its block
    output equals the BF16 block's bit for bit.  Grouping down along I instead would mix
    the columns' scales inside a group and move the weights."""
    rng = np.random.default_rng(4)
    d, inter, E = 128, 64, 2

    def grid_rows(n, exp0):
        return np.stack([np.concatenate([_grid_group(rng, exp0 - (i % 3))[0]
                                         for _ in range(d // 64)]) for i in range(n)])

    gate = np.stack([grid_rows(inter, -5) for _ in range(E)])
    up = np.stack([grid_rows(inter, -5) for _ in range(E)])
    down = np.stack([grid_rows(inter, -6).T for _ in range(E)])   # columns on the grid
    router = _bf16(rng.normal(0, 0.05, (d, E)))
    base = oracle.ArrayLayer(gate, up, down, router)
    lay = q4.Q4Layer(base)
    for e in range(E):
        for a, b in zip(lay.expert(e)[:3], base.expert(e)[:3]):
            np.testing.assert_array_equal(a, b)
    # the same down grouped along I does move
    moved = q4.dequantize_groups(*q4.quantize_groups(down[0]))
    assert np.abs(moved - down[0]).max() > 0
    x = _bf16(rng.normal(0, 1, (3, d)))
    r0 = oracle.moe_block(x, base, top_e=2, k=20)
    r1 = oracle.moe_block(x, lay, top_e=2, k=20)
    np.testing.assert_array_equal(r0["y"], r1["y"])


def test_q4_block_stays_near_the_bf16_block():
    """On Gaussian weights the 4-bit dense block differs from the BF16 one by the
    quantisation noise: a group of 64 spans about 4.8 sigma, so the step is ~0.32 sigma
    and the rounding error ~0.09 sigma (uniform, step / sqrt(12)) per weight; gate.x,
    up.x and the down product each carry ~9 % relative noise, ~15 % on the output."""
    w = synth.TINY
    base = oracle.SynthLayer(w)
    lay = q4.Q4Layer(base)
    x = synth.activations(w, step=0)
    y0 = oracle.dense_moe(x, base, w.top_e)["y"]
    y1 = oracle.dense_moe(x, lay, w.top_e)["y"]
    rel = np.linalg.norm(y1 - y0) / np.linalg.norm(y0)
    assert 0.08 < rel < 0.25


def test_record_and_read_bytes():
    assert q4.record_bytes(2048) == 3 * 1024 + 3 * 32 * 4 == 3456
    assert q4.record_bytes(64) == 112          # 96 + 12 = 108, padded to 16 bytes
    # Qwen3-30B-A3B-shaped block, batch 1, k = 138, r = 32: per expert
    # 138 * 3456 (records) + 768 * 2048 / 4 (sketch) + 4 * 768 (alpha) + 4 * 2048 * 32
    assert q4.read_bytes([138] * 8, 2048, 768, 32) == 8 * (476_928 + 393_216 + 3_072 + 262_144)
    assert q4.read_bytes([138] * 8, 2048, 768, 32) == 9_082_880
