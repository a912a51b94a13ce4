"""The numpy oracle against a second, independently written restatement in plain C99
(``oracle/c/msb_oracle.c``, FP64 loops).  Both follow the same readings; they share no
code.  Agreement pins the numpy oracle's implementation (an index, a transposed
operand, a dropped term would differ) beyond its closed-form and brute-force pins.

Routing and kept sets must match exactly, except channels whose scores lie within
1e-12 (relative) of the k-th score (the two sum in different orders); outputs within
1e-10 relative L2 per token (FP64 rounding only).
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import c_oracle

SEL_EPS = 1e-12
Y_RTOL = 1e-10


def _both(w, x_bits, lw=None, k=None, mode="topk", tau=0.0, renorm=True, rank=True):
    lw = synth.layer_weights(w) if lw is None else lw
    a, b = (lw.lr_a, lw.lr_b) if rank and w.rank else (None, None)
    lay = oracle.ArrayLayer(lw.gate, lw.up, lw.down, lw.router, a, b)
    k = w.k if k is None else k
    ref = oracle.moe_block(x_bits, lay, w.top_e, k, renorm=renorm, mode=mode, tau=tau)
    got = c_oracle.moe_block(x_bits, lw.gate, lw.up, lw.down, lw.router, w.top_e, k=k, lr_a=a,
                             lr_b=b, renorm=renorm, mode=mode, tau=tau)
    return ref, got


def _agree(ref, got, k=None, mode="topk"):
    np.testing.assert_array_equal(got["ids"], ref["ids"])
    np.testing.assert_allclose(got["w"], ref["w"], rtol=1e-13)
    for key, s_ref in ref["sel"].items():
        s_got = got["sel"][key]
        if mode != "dense":
            np.testing.assert_allclose(got["scores"][key], ref["scores"][key], rtol=1e-12,
                                       atol=1e-14 * np.abs(ref["scores"][key]).max())
        if np.array_equal(s_got, s_ref):
            continue
        assert mode == "topk", (key, "threshold/dense sets differ")
        sc = ref["scores"][key]
        kth = np.sort(sc)[::-1][k - 1]
        diff = np.setxor1d(s_got, s_ref)
        assert len(s_got) == len(s_ref) == k
        assert np.all(np.abs(sc[diff] - kth) <= SEL_EPS * kth), (key, diff)
    for t in range(ref["y"].shape[0]):
        yr, yg = ref["y"][t], got["y"][t]
        assert np.linalg.norm(yg - yr) <= Y_RTOL * np.linalg.norm(yr), t


def test_tiny_block_every_step_kind():
    w = synth.TINY
    lw = synth.layer_weights(w)
    x = np.concatenate([synth.activations(w, s) for s in range(4)])
    ref, got = _both(w, x, lw)
    _agree(ref, got, w.k)
    ref, got = _both(w, x, lw, mode="dense", rank=False)
    _agree(ref, got, mode="dense")
    ref_topk, _ = _both(w, x[:1], lw)             # tau from the scores of one token
    tau = float(np.quantile(np.concatenate(list(ref_topk["scores"].values())), 0.85))
    ref, got = _both(w, x, lw, mode="threshold", tau=tau)
    _agree(ref, got, mode="threshold")


def test_qwen_shaped_block():
    """d = 2048, I = 768, top-8, k = 138, r = 32, heavy rows; 16 of the 128 experts."""
    w = synth.QWEN30B_BLOCK.with_(experts=16)
    lw = synth.layer_weights(w)
    x = synth.activations(w, 0, batch=2)
    ref, got = _both(w, x, lw)
    _agree(ref, got, w.k)


def test_exact_ties_and_zero_rows():
    """Duplicated gate rows give bit-equal scores in both; zero rows score 0: the tie
    rule (lower index first) must pick the same channels in both."""
    w = synth.TINY.with_(d=64, inter=48, experts=2, top_e=2, k=20, rank=0, seed=5)
    lw = synth.layer_weights(w)
    for e in range(2):
        lw.gate[e, 10:20] = lw.gate[e, 0]
        lw.gate[e, 30:40] = 0
    x = synth.activations(w, 1, batch=3)
    for k in (1, 5, 11, 20, 38, 47, 48):
        ref, got = _both(w, x, lw, k=k)
        for key in ref["sel"]:
            np.testing.assert_array_equal(got["sel"][key], ref["sel"][key])
        _agree(ref, got, k)


@pytest.mark.parametrize("renorm", [True, False])
def test_router_renormalisation(renorm):
    w = synth.TINY.with_(experts=8, top_e=3)
    lw = synth.layer_weights(w)
    x = synth.activations(w, 2, batch=2)
    ref, got = _both(w, x, lw, renorm=renorm)
    _agree(ref, got, w.k)
    assert np.allclose(got["w"].sum(axis=1), 1.0) == renorm
