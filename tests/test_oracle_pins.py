"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each test checks it against a
hand-worked example (tests/golden), a closed form, brute force, or a special
case with a textbook value.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MATH = {"log": math.log, "exp": math.exp, "sqrt": math.sqrt, "e": math.e}


def ev(s):
    return float(eval(str(s), {"__builtins__": {}}, MATH))


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def closed_form_layer(g):
    E = g["dims"]["E"]
    gate = np.array([g["gate"][str(e)] for e in range(E)], dtype=np.float64)
    up = np.array([g["up"][str(e)] for e in range(E)], dtype=np.float64)
    down = np.array([g["down_d_by_I"][str(e)] for e in range(E)], dtype=np.float64)
    a = np.array([g["lowrank_A_d_by_r"][str(e)] for e in range(E)], dtype=np.float64)
    b = np.array([g["lowrank_B_r_by_d"][str(e)] for e in range(E)], dtype=np.float64)
    router = np.array(g["router_d_by_E"], dtype=np.float64)
    return oracle.ArrayLayer(gate, up, down, router, a, b)


# ----------------------------------------------------------------------------- closed-form block

@pytest.mark.parametrize("renorm", [True, False])
def test_closed_form_block(renorm):
    g = load("closed_form_block.json")
    lay = closed_form_layer(g)
    x = np.array([[ev(v) for v in g["x"]]])
    dims = g["dims"]
    res = oracle.moe_block(x, lay, top_e=dims["top_e"], k=dims["k"], renorm=renorm)
    ex = g["expect"]
    assert list(res["ids"][0]) == ex["ids"]
    w_expect = [ev(v) for v in (ex["w_renorm"] if renorm else ex["w_plain"])]
    np.testing.assert_allclose(res["w"][0], w_expect, rtol=1e-14)
    for e, sel in ex["sel"].items():
        assert list(res["sel"][(0, int(e))]) == sel
        np.testing.assert_allclose(res["scores"][(0, int(e))], [ev(v) for v in ex["scores"][e]],
                                   rtol=1e-14, atol=1e-15)
    y_expect = [ev(v) for v in (ex["y_renorm"] if renorm else ex["y_plain"])]
    np.testing.assert_allclose(res["y"][0], y_expect, rtol=1e-13, atol=1e-14)


def test_closed_form_dense_block():
    g = load("closed_form_block.json")
    lay = closed_form_layer(g)
    x = np.array([[ev(v) for v in g["x"]]])
    res = oracle.dense_moe(x, lay, top_e=2, renorm=True)
    np.testing.assert_allclose(res["y"][0], [ev(v) for v in g["expect"]["y_dense_renorm"]],
                               rtol=1e-13, atol=1e-13)
    # The sparse block at k = I with rank 0 is the dense block.
    sp = oracle.moe_block(x, lay, top_e=2, k=3, renorm=True, rank=0)
    np.testing.assert_array_equal(sp["y"], res["y"])


def test_rank_zero_drops_lowrank_exactly():
    g = load("closed_form_block.json")
    lay = closed_form_layer(g)
    x = np.array([[ev(v) for v in g["x"]]])
    full = oracle.moe_block(x, lay, top_e=2, k=2, renorm=True)
    r0 = oracle.moe_block(x, lay, top_e=2, k=2, renorm=True, rank=0)
    # y2 loses 3/4 * [0,0,1,0], y3 loses 1/4 * [0,0,0,2 log 3]
    np.testing.assert_allclose(full["y"][0] - r0["y"][0], [0, 0, 0.75, 0.5 * math.log(3)],
                               rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------- sketch

def test_sketch_hand_rows():
    g = load("sketch_rows.json")
    for row in g["rows"]:
        w = np.array([[ev(v) for v in row["w"]]])
        t, alpha = oracle.ternary_sketch(w)
        assert list(t[0]) == row["T"], row["why"]
        assert alpha.dtype == np.float32
        assert alpha[0] == np.float32(ev(row["alpha"])), row["why"]


def test_sketch_gaussian_closed_form():
    g = load("sketch_rows.json")["gaussian"]
    tt = 0.7 * math.sqrt(2 / math.pi)
    kept = math.erfc(tt / math.sqrt(2))
    ratio = math.exp(-tt * tt / 2) / math.sqrt(2 * math.pi) / (0.5 * math.erfc(tt / math.sqrt(2)))
    assert abs(kept - g["kept_fraction"]) < 1e-5
    assert abs(ratio - g["alpha_over_sigma"]) < 1e-4
    rng = np.random.default_rng(1234)
    d = 1 << 18
    for sigma in (0.02, 0.08):
        w = rng.standard_normal((4, d)) * sigma
        t, alpha = oracle.ternary_sketch(w)
        frac = np.count_nonzero(t, axis=1) / d
        np.testing.assert_allclose(frac, kept, atol=4 / math.sqrt(d))
        np.testing.assert_allclose(alpha / sigma, ratio, rtol=3e-3)


def test_sketch_scale_invariance_of_heavy_rows():
    # Scaling a row by 4 scales delta and alpha by 4 and keeps T (all exact in binary).
    rng = np.random.default_rng(7)
    w = np.round(rng.standard_normal((8, 512)) * 64) / 64
    t1, a1 = oracle.ternary_sketch(w)
    t4, a4 = oracle.ternary_sketch(4 * w)
    np.testing.assert_array_equal(t1, t4)
    np.testing.assert_array_equal(a4, 4 * a1)


def test_scores_hand():
    t = np.array([[1, 0, -1, 1], [0, 0, 0, 0], [-1, -1, -1, -1]], dtype=np.int8)
    alpha = np.array([0.5, 3.0, 0.25], dtype=np.float32)
    x = np.array([2.0, 7.0, 1.0, -4.0])
    # row0: |2 - 1 - 4| * 0.5 = 1.5; row1: 0; row2: |-(2+7+1-4)| * 0.25 = 1.5
    np.testing.assert_array_equal(oracle.channel_scores(t, alpha, x), [1.5, 0.0, 1.5])


# ----------------------------------------------------------------------------- selection

def _brute_topk(s, k):
    """The unique k-subset whose every member beats every non-member by (score desc, index asc)."""
    n = len(s)
    found = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j)
                 for i in inside for j in range(n) if j not in inside)
        if ok:
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


def test_topk_vs_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(300):
        n = int(rng.integers(1, 11))
        k = int(rng.integers(1, n + 1))
        s = rng.integers(0, 4, size=n).astype(np.float64)   # many ties
        assert list(oracle.topk_channels(s, k)) == _brute_topk(list(s), k)
    for trial in range(50):
        n = int(rng.integers(1, 9))
        s = rng.random(n)
        for k in range(1, n + 1):
            assert list(oracle.topk_channels(s, k)) == _brute_topk(list(s), k)


def test_topk_budget_is_exact():
    rng = np.random.default_rng(5)
    for _ in range(20):
        s = rng.integers(0, 3, size=64).astype(float)
        for k in (1, 17, 63, 64):
            sel = oracle.topk_channels(s, k)
            assert sel.size == k and np.all(np.diff(sel) > 0)


def test_threshold_selector():
    s = np.array([0.5, 2.0, 1.0, 3.0, 1.0])
    assert list(oracle.threshold_channels(s, 1.0)) == [1, 3]        # strict
    assert list(oracle.threshold_channels(s, 0.0)) == [0, 1, 2, 3, 4]
    assert list(oracle.threshold_channels(s, 3.0)) == []
    # With distinct scores, tau = the (k+1)-th largest score reproduces top-k.
    rng = np.random.default_rng(11)
    v = rng.random(40)
    for k in (1, 7, 39):
        tau = np.sort(v)[::-1][k]
        assert list(oracle.threshold_channels(v, tau)) == list(oracle.topk_channels(v, k))


def test_calibrate_threshold():
    scores = np.arange(1, 101, dtype=float)          # 1..100
    tau = oracle.calibrate_threshold(scores, 0.18)   # m = 18 -> 19th largest = 82
    assert tau == 82.0
    assert np.count_nonzero(scores > tau) == 18


# ----------------------------------------------------------------------------- router

def test_router_softmax_closed_form_and_ties():
    # logits [ln1, ln2, ln3, ln4] -> p = [1,2,3,4]/10
    w_router = np.diag([0.0, math.log(2), math.log(3), math.log(4)])
    x = np.ones(4)
    ids, w, logits = oracle.route(x, w_router, top_e=2, renorm=False)
    assert list(ids) == [3, 2]
    np.testing.assert_allclose(w, [0.4, 0.3], rtol=1e-14)
    ids, w, _ = oracle.route(x, w_router, top_e=2, renorm=True)
    np.testing.assert_allclose(w, [4 / 7, 3 / 7], rtol=1e-14)
    # ties: equal logits rank by lower expert index
    ids, w, _ = oracle.route(np.ones(4), np.zeros((4, 4)), top_e=3, renorm=False)
    assert list(ids) == [0, 1, 2]
    np.testing.assert_allclose(w, [0.25] * 3)


# ----------------------------------------------------------------------------- expert pieces

def test_expert_swiglu_special_values():
    d = 3
    x = np.array([math.log(3), 0.0, 1.0])
    gate = np.array([[1.0, 0, 0], [0, 5.0, 0], [-1.0, 0, 0]])   # g = ln3, 0, -ln3
    up = np.array([[0, 0, 2.0], [0, 0, 9.0], [0, 0, 4.0]])      # u = 2, 9, 4
    down = np.eye(d)
    y = oracle.expert_output(x, gate, up, down, [0, 1, 2])
    # silu(ln3)*2 = 1.5 ln3 ; silu(0)*9 = 0 ; silu(-ln3)*4 = -ln3
    np.testing.assert_allclose(y, [1.5 * math.log(3), 0.0, -math.log(3)], rtol=1e-14, atol=1e-15)
    y = oracle.expert_output(x, gate, up, down, [2])
    np.testing.assert_allclose(y, [0, 0, -math.log(3)], rtol=1e-14, atol=1e-15)


def test_lowrank_term():
    a = np.array([[1.0, 0.0], [0.0, 2.0], [0.0, 0.0]])     # d=3, r=2
    b = np.array([[0.0, 1.0, 0.0], [1.0, 0.0, 1.0]])       # r=2, d=3
    x = np.array([3.0, 5.0, 7.0])
    # B x = [5, 10]; A (B x) = [5, 20, 0]
    np.testing.assert_array_equal(oracle.lowrank_term(x, a, b), [5.0, 20.0, 0.0])
    np.testing.assert_array_equal(oracle.lowrank_term(x, a[:, :0], b[:0]), [0, 0, 0])


def test_single_expert_dense_is_swiglu_ffn():
    # E = K = 1, k = I, no low-rank: the block is the SwiGLU FFN
    # y = W_down (silu(W_gate x) * (W_up x)); checked with torch's silu on CPU.
    import torch
    rng = np.random.default_rng(2)
    d, I = 16, 12
    gate, up = rng.standard_normal((1, I, d)), rng.standard_normal((1, I, d))
    down = rng.standard_normal((1, d, I))
    router = rng.standard_normal((d, 1))
    x = rng.standard_normal((1, d))
    lay = oracle.ArrayLayer(gate, up, down, router)
    y = oracle.moe_block(x, lay, top_e=1, k=I, renorm=True, rank=0)["y"][0]
    tx = torch.tensor(x[0])
    ref = torch.tensor(down[0]) @ (torch.nn.functional.silu(torch.tensor(gate[0]) @ tx)
                                    * (torch.tensor(up[0]) @ tx))
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("renorm", [True, False])
def test_all_experts_dense_is_softmax_weighted_ffns(renorm):
    # K = E, k = I, no low-rank: every expert is used densely and the block is
    # sum_e softmax(x W_router)_e * FFN_e(x) (with K = E renormalisation changes nothing);
    # checked with torch's softmax and silu on CPU.
    import torch
    rng = np.random.default_rng(8)
    d, I, E = 16, 10, 5
    gate, up = rng.standard_normal((E, I, d)), rng.standard_normal((E, I, d))
    down = rng.standard_normal((E, d, I))
    router = rng.standard_normal((d, E))
    x = rng.standard_normal((2, d))
    lay = oracle.ArrayLayer(gate, up, down, router)
    y = oracle.moe_block(x, lay, top_e=E, k=I, renorm=renorm, rank=0)["y"]
    for t in range(2):
        tx = torch.tensor(x[t])
        p = torch.softmax(tx @ torch.tensor(router), dim=0)
        ref = sum(p[e] * (torch.tensor(down[e]) @ (torch.nn.functional.silu(torch.tensor(gate[e]) @ tx)
                                                  * (torch.tensor(up[e]) @ tx))) for e in range(E))
        np.testing.assert_allclose(y[t], ref.numpy(), rtol=1e-11, atol=1e-11)


# ----------------------------------------------------------------------------- numbers, glue

def test_round_to_bf16():
    one = 1.0
    cases = {one + 2 ** -8: 1.0,                    # tie -> even (1.0)
             one + 3 * 2 ** -8: one + 2 * 2 ** -7,  # tie -> even
             one + 2 ** -8 + 2 ** -20: one + 2 ** -7,
             -3.0: -3.0, 0.0: 0.0}
    for v, r in cases.items():
        assert oracle.round_to_bf16(v) == r
    # against the generator's independent float32 -> bf16 bit rounding
    rng = np.random.default_rng(0)
    v = rng.standard_normal(10000).astype(np.float32)
    np.testing.assert_array_equal(oracle.round_to_bf16(v.astype(np.float64)),
                                  oracle.bf16_to_f64(synth.f32_to_bf16_bits(v)))


def test_rmsnorm_and_stack_layer():
    h = np.array([[1.0, -1.0, 1.0, -1.0], [3.0, 4.0, 0.0, 0.0]])
    r = oracle.rmsnorm(h, eps=0.0)
    np.testing.assert_allclose(r[0], [1, -1, 1, -1], rtol=1e-15)
    np.testing.assert_allclose(r[1], np.array([3.0, 4.0, 0, 0]) / math.sqrt(25 / 4), rtol=1e-15)
    # residual: h_next = h + block(BF16(RMSNorm(h))) on the closed-form block
    g = load("closed_form_block.json")
    lay = closed_form_layer(g)
    h0 = np.array([[1.0, 1.0, -1.0, 1.0]])   # RMSNorm(h0) = h0 (eps aside), exact in BF16
    h1, x_used, res = oracle.stack_layer(h0, lay, top_e=2, k=2, eps=0.0)
    np.testing.assert_array_equal(x_used, h0)
    np.testing.assert_allclose(h1, h0 + res["y"], rtol=0, atol=0)


def test_read_bytes_fixed_budget():
    # d=2048, I=768, r=32, 8 experts of 138 channels each (one token):
    per_expert = 768 * 2048 // 4 + 4 * 768 + 6 * 2048 * 138 + 4 * 2048 * 32
    assert oracle.read_bytes([138] * 8, 2048, 768, 32) == 8 * per_expert == 18833408
    assert oracle.read_bytes([768] * 8, 2048, 768, 0, dense=True) == 75497472


def test_tiny_workload_budget_invariant():
    """Fixed read volume: on the tiny workload every (token, expert) keeps exactly k
    channels, so every step reads the same channel bytes K * k * 6d."""
    w = synth.TINY
    lay = oracle.SynthLayer(w)
    for step in range(4):
        x = synth.activations(w, step)
        res = oracle.moe_block(x, lay, w.top_e, w.k)
        assert len(res["sel"]) == w.top_e
        sizes = [len(v) for v in res["sel"].values()]
        assert sizes == [w.k] * w.top_e
        assert sum(sizes) * 6 * w.d == w.top_e * w.k * 6 * w.d


# ----------------------------------------------------------------------------- generator

def test_budget_to_k_reproduces_every_stated_k():
    """k = round(budget * I): the 18 % and 13 % budgets of I = 768 give the workloads'
    k = 138 and 100, 18 % of I = 1536 gives 276; 100 % is every channel."""
    assert synth.budget_k(0.18, 768) == 138 == synth.QWEN30B_BLOCK.k
    assert synth.budget_k(0.13, 768) == 100 == synth.QWEN30B_BLOCK_13.k
    assert synth.budget_k(0.18, 1536) == 276 == synth.LARGE_BLOCK.k
    assert synth.budget_k(1.0, 768) == 768


def test_generator_determinism_and_shapes():
    w = synth.TINY
    a = synth.expert_gate(w, 3)
    assert a.shape == (w.inter, w.d) and a.dtype == np.uint16
    np.testing.assert_array_equal(a, synth.expert_gate(w, 3))
    assert not np.array_equal(a, synth.expert_gate(w, 4))
    assert not np.array_equal(a, synth.expert_up(w, 3))
    assert synth.expert_down(w, 0).shape == (w.d, w.inter)
    x0 = synth.activations(w, 0)
    assert x0.shape == (1, w.d)
    assert not np.array_equal(x0, synth.activations(w, 1))
    assert not np.array_equal(synth.activations(w, 0, 4)[0],
                              synth.calibration_activations(w, 0, 4)[0])


def test_generator_heavy_rows():
    w = synth.QWEN30B_BLOCK.with_(d=256, experts=2)
    rows = synth.heavy_rows(w, 1)
    assert rows.size == round(0.05 * w.inter) and np.all(np.diff(rows) > 0)
    g = synth.bf16_bits_to_f32(synth.expert_gate(w, 1)).astype(np.float64)
    std = g.std(axis=1)
    heavy = np.zeros(w.inter, bool)
    heavy[rows] = True
    assert abs(std[heavy].mean() / std[~heavy].mean() - 4.0) < 0.1
    assert abs(std[~heavy].mean() - w.sigma) < 0.001
