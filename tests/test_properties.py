"""Property-based checks (hypothesis) of the oracle's invariants and of the host packers
against the oracle, on random small inputs.  CPU only.

Invariants follow from the definitions the oracle restates: the ternary sketch keeps
exactly the entries above 0.7 * mean|W| and its scale is their mean magnitude; top-k
returns k distinct ascending channels, none outscored by a channel left out, ties
broken towards the lower index; the router's kept weights sum to one with
renormalisation; the 4-bit quantiser's codes are the nearest of the 16 on its grid.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
import synth
from oracle import q4

SETTINGS = settings(max_examples=60, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])


def _bf16_rows(seed, n, d, scale):
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, scale, (n, d))
    w[rng.random((n, d)) < 0.1] = 0.0                  # exact zeros
    return oracle.round_to_bf16(w)


@SETTINGS
@given(seed=st.integers(0, 2**32 - 1), n=st.integers(1, 6), d=st.sampled_from([8, 64, 192]),
       scale=st.sampled_from([1e-3, 0.02, 1.0, 300.0]))
def test_sketch_invariants(seed, n, d, scale):
    w = _bf16_rows(seed, n, d, scale)
    t, alpha = oracle.ternary_sketch(w)
    delta = 0.7 * np.abs(w).mean(axis=1, keepdims=True)
    kept = t != 0
    assert set(np.unique(t)) <= {-1, 0, 1}
    np.testing.assert_array_equal(kept, np.abs(w) > delta)
    np.testing.assert_array_equal(t[kept], np.sign(w[kept]))
    for i in range(n):
        if kept[i].any():
            assert alpha[i] == np.float32(np.abs(w[i][kept[i]]).mean())
            assert alpha[i] >= np.float32(delta[i, 0])
        else:
            assert alpha[i] == 0.0


@SETTINGS
@given(seed=st.integers(0, 2**32 - 1), n=st.integers(1, 80), levels=st.integers(1, 12),
       data=st.data())
def test_topk_invariants(seed, n, levels, data):
    k = data.draw(st.integers(1, n))
    rng = np.random.default_rng(seed)
    s = rng.integers(0, levels, n).astype(np.float64)   # few levels: many ties
    sel = oracle.topk_channels(s, k)
    assert len(sel) == k and len(set(sel.tolist())) == k
    assert np.all(np.diff(sel) > 0)
    out = np.setdiff1d(np.arange(n), sel)
    if out.size:
        assert s[sel].min() >= s[out].max()
        # ties at the boundary go to the lower index
        kth = s[sel].min()
        assert np.all(out[s[out] == kth] > sel[s[sel] == kth].max())


@SETTINGS
@given(seed=st.integers(0, 2**32 - 1), E=st.integers(1, 16), data=st.data())
def test_router_invariants(seed, E, data):
    K = data.draw(st.integers(1, E))
    rng = np.random.default_rng(seed)
    d = 16
    x = rng.normal(size=d)
    wr = rng.normal(size=(d, E))
    ids, w, logits = oracle.route(x, wr, K, renorm=True)
    assert len(set(ids.tolist())) == K
    assert np.isclose(w.sum(), 1.0)
    assert np.all(np.diff(logits[ids]) <= 0)            # rank order
    rest = np.setdiff1d(np.arange(E), ids)
    if rest.size:
        assert logits[ids].min() >= logits[rest].max()
    _, w0, _ = oracle.route(x, wr, K, renorm=False)
    p = np.exp(logits - logits.max())
    np.testing.assert_allclose(w0, p[ids] / p.sum())


@SETTINGS
@given(seed=st.integers(0, 2**32 - 1), groups=st.integers(1, 4),
       scale=st.sampled_from([1e-3, 0.02, 1.0, 300.0]), shift=st.sampled_from([0.0, 1.0, -40.0]))
def test_q4_codes_are_nearest(seed, groups, scale, shift):
    w = _bf16_rows(seed, 3, 64 * groups, scale) + oracle.round_to_bf16(shift)
    w = oracle.round_to_bf16(w)
    q, s, b = q4.quantize_groups(w)
    g = w.reshape(3, groups, 64)
    cand = s[..., None, None] * np.arange(16.0) + b[..., None, None]
    dist = np.abs(g[..., None] - cand)
    chosen = np.take_along_axis(dist, q.reshape(g.shape)[..., None].astype(np.int64), -1)[..., 0]
    np.testing.assert_array_equal(chosen, dist.min(-1))
    assert np.all(np.abs(w - q4.dequantize_groups(q, s, b)).reshape(g.shape)
                  <= s[..., None] / 2 * (1 + 1e-12))


@pytest.fixture(scope="module")
def msb():
    from token_top_expert_b200 import build
    build.build()
    import token_top_expert_b200 as m
    m.load_library()
    return m


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), d=st.sampled_from([64, 128, 320]), inter=st.integers(1, 40),
       experts=st.integers(1, 3), heavy=st.sampled_from([0.0, 0.2]))
def test_packers_match_the_oracle_on_random_layers(msb, seed, d, inter, experts, heavy):
    from test_host import decode_q4_records, decode_sketch
    w = synth.TINY.with_(d=d, inter=inter, experts=experts, top_e=1, rank=0, seed=seed,
                         heavy_frac=heavy, heavy_scale=4.0)
    lw = synth.layer_weights(w)
    dims = msb.Dims(d, inter, experts, 1, 0)
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims, threads=2)
    pq = msb.pack_q4(lw.gate, lw.up, lw.down, lw.router, dims, threads=2)
    for e in range(experts):
        g = oracle.bf16_to_f64(lw.gate[e])
        t, a = oracle.ternary_sketch(g)
        np.testing.assert_array_equal(decode_sketch(pk["sketch"], dims, e)[:inter], t)
        np.testing.assert_array_equal(pk["alpha"][e, :inter], a)
        q, s, b, pad = decode_q4_records(pq["records"][e], d)
        assert not pad.any()
        for part, mat in enumerate((lw.gate[e], lw.up[e], lw.down[e].T)):
            q_ref, s_ref, b_ref = q4.quantize_groups(oracle.bf16_to_f64(mat))
            np.testing.assert_array_equal(q[:, part], q_ref)
            np.testing.assert_array_equal(s[:, part], s_ref)
            np.testing.assert_array_equal(b[:, part], b_ref)
        gq = q4.q4_weights(g, oracle.bf16_to_f64(lw.up[e]), oracle.bf16_to_f64(lw.down[e]))[0]
        tq, aq = oracle.ternary_sketch(gq)
        np.testing.assert_array_equal(decode_sketch(pq["sketch"], dims, e)[:inter], tq)
        np.testing.assert_array_equal(pq["alpha"][e, :inter], aq)


def test_calibrate_threshold_matches_oracle():
    """The package's threshold calibration (selection) and the oracle's (sort) agree,
    with and without ties, at budgets 0, 13%, 18%, 100%."""
    import oracle
    from token_top_expert_b200.block import calibrate_threshold
    rng = np.random.default_rng(5)
    for scores in (rng.random(4096), np.round(rng.random(4096) * 20) / 20, np.ones(7), rng.random(1)):
        for budget in (0.0, 0.13, 0.18, 1.0):
            assert calibrate_threshold(scores, budget) == oracle.calibrate_threshold(scores, budget)
