"""Weight-derived low-rank compensation (host-side weight preparation).

Pinned against the oracle's restatement of the selection (sketch, scores, top-k), against
a closed form (orthogonal gate/up rows of channels that are always skipped: the map's
coefficient is E[a sigmoid(a)] for a ~ N(0, |gate_j|^2), evaluated here by quadrature),
and against the defining properties of the construction: nothing skipped gives a zero map;
on fresh samples from the prior the compensated error is not larger than the uncompensated
one; the factors are the leading singular directions of the map (Eckart-Young).
"""
import numpy as np
import pytest

import oracle
from token_top_expert_b200 import lowrank


def _expert(d, inter, seed, scale):
    rng = np.random.default_rng(seed)
    return (rng.normal(0, scale, (inter, d)), rng.normal(0, scale, (inter, d)),
            rng.normal(0, scale, (d, inter)))


def test_sketch_is_the_packers_rule():
    """The estimate's sketch comes from the packer (msb_ternary_rows); it equals the
    oracle's ternarisation, including entries exactly at the 0.7 mean |W| threshold
    (strict inequality: not kept), signs, and an all-zero row (alpha 0)."""
    rng = np.random.default_rng(9)
    w = rng.normal(0, 0.02, (24, 80)).astype(np.float32)
    w[3] = 0.0
    w[5] = 1.0
    w[5, :20] = 5.0   # mean |W| = 2, threshold 1.4: the 1.0 entries drop, the 5.0 stay
    w[6, :40] = 13.0  # mean |W| = 10, threshold exactly 7: the 7.0 entries are not kept
    w[6, 40:] = 7.0
    w[7] = -w[6]
    t, alpha = lowrank._ternary(w)
    rt, ra = oracle.ternary_sketch(w.astype(np.float64))
    np.testing.assert_array_equal(t, rt)
    np.testing.assert_allclose(alpha, ra, rtol=1e-6, atol=0)
    assert alpha[3] == 0.0 and (t[3] == 0).all()
    assert (t[5, :20] == 1).all() and (t[5, 20:] == 0).all() and alpha[5] == 5.0
    assert (t[6, :40] == 1).all() and (t[6, 40:] == 0).all() and alpha[6] == 13.0
    assert (t[7, :40] == -1).all() and (t[7, 40:] == 0).all() and alpha[7] == 13.0
    with pytest.raises(ValueError):
        lowrank._ternary(np.zeros((0, 8), np.float32))


def test_channel_moments_match_the_oracle_selection():
    d, inter, k = 64, 48, 12
    gate, up, down = _expert(d, inter, 1, 0.2)
    x = np.random.default_rng(2).standard_normal((40, d)).astype(np.float32)
    ma, mb = lowrank.channel_moments(gate, up, down, k, x)
    t, alpha = oracle.ternary_sketch(gate)
    ra, rb = np.zeros(inter), np.zeros(inter)
    for xi in x.astype(np.float64):
        keep = oracle.topk_channels(oracle.channel_scores(t, alpha, xi), k)
        a, b = gate @ xi, up @ xi
        h = a / (1.0 + np.exp(-a)) * b
        h[keep] = 0.0
        ra += h * a
        rb += h * b
    np.testing.assert_allclose(ma, ra / len(x), rtol=1e-3, atol=1e-6)
    np.testing.assert_allclose(mb, rb / len(x), rtol=1e-3, atol=1e-6)


def test_orthogonal_rows_closed_form():
    """Channel 0 has a dominant gate row, so with k = 1 channels 1..3 are always skipped.
    Their gate and up rows lie on distinct axes, so b is independent of a and of
    the selection: E[h a] = 0 and E[h b] = E[silu(a)] |up|^2, hence c_a = 0 and
    c_b = E[silu(a)] = E[a sigmoid(a)], a ~ N(0, |gate_j|^2)."""
    d, inter = 16, 4
    gate, up, down = np.zeros((inter, d)), np.zeros((inter, d)), np.zeros((d, inter))
    gate[0, 0] = 50.0
    up[0, 1] = 1.0
    sig = [0.0, 0.7, 1.3, 2.0]
    for j in range(1, inter):
        gate[j, 2 * j] = sig[j]
        up[j, 2 * j + 1] = 0.5
        down[j, j] = 1.0
    x = np.random.default_rng(5).standard_normal((400_000, d)).astype(np.float32)
    ma, mb = lowrank.channel_moments(gate, up, down, 1, x)
    m = lowrank.structured_map(gate, up, down, ma, mb)
    z = np.linspace(-12, 12, 24001)
    phi = np.exp(-z * z / 2) / np.sqrt(2 * np.pi)
    for j in range(1, inter):
        a = sig[j] * z
        expect = np.trapezoid(a / (1 + np.exp(-a)) * phi, z)   # E[silu(a)]
        # M[j] = c_a gate_j + c_b up_j with up_j = 0.5 e_(2j+1)
        assert m[j, 2 * j + 1] == pytest.approx(0.5 * expect, rel=0.03)
        assert abs(m[j, 2 * j]) < 0.03 * abs(expect)
    assert np.all(m[0] == 0.0)  # channel 0 is never skipped


def test_nothing_skipped_gives_a_zero_map():
    d, inter = 32, 24
    gate, up, down = _expert(d, inter, 3, 0.2)
    a, b = lowrank.derive_lowrank(gate[None], up[None], down[None], k=inter, rank=4, samples=256)
    assert not a.any() and not b.any()


def test_compensation_does_not_add_error_on_fresh_samples():
    d, inter, k, r = 64, 96, 18, 8
    gate, up, down = _expert(d, inter, 5, 0.15)
    a, b = lowrank.derive_lowrank(gate[None], up[None], down[None], k=k, rank=r, samples=8192,
                                  seed=11)
    af, bf = oracle.bf16_to_f64(a[0]), oracle.bf16_to_f64(b[0])
    t, alpha = oracle.ternary_sketch(gate)
    xs = np.random.default_rng(99).standard_normal((400, d))
    e0 = e1 = 0.0
    for x in xs:
        keep = oracle.topk_channels(oracle.channel_scores(t, alpha, x), k)
        skipped = np.setdiff1d(np.arange(inter), keep)
        y = oracle.expert_output(x, gate, up, down, skipped)
        e0 += float(y @ y)
        res = y - af @ (bf @ x)
        e1 += float(res @ res)
    assert e1 < e0
    print("skipped-channel error kept by the compensation: %.4f" % (e1 / e0))


def test_factors_are_the_leading_singular_directions():
    d, inter, k, r = 48, 40, 10, 6
    gate, up, down = _expert(d, inter, 7, 0.2)
    x = np.random.default_rng([4, 0]).standard_normal((1024, d), dtype=np.float32)
    ma, mb = lowrank.channel_moments(gate, up, down, k, x)
    m = lowrank.structured_map(gate, up, down, ma, mb)
    a, b = lowrank.derive_lowrank(gate[None], up[None], down[None], k=k, rank=r, samples=1024,
                                  seed=4, chunk=1024)
    s = np.linalg.svd(m, compute_uv=False)
    resid = np.linalg.norm(m - oracle.bf16_to_f64(a[0]) @ oracle.bf16_to_f64(b[0]))
    tail = np.sqrt((s[r:] ** 2).sum())
    # Eckart-Young, up to the BF16 rounding of the factors
    assert resid == pytest.approx(tail, rel=0.05, abs=1e-2 * s[0])


def test_leading_factors_of_a_product():
    """With n < d the SVD of the n x n QR core gives the singular values and the rank-r
    truncation of p @ q that a direct SVD of the d x d product gives; asking for more
    triplets than the product's rank pads with zeros."""
    rng = np.random.default_rng(9)
    d, n, r = 80, 24, 6
    p, q = rng.normal(size=(d, n)), rng.normal(size=(n, d))
    u, s, vt = lowrank.leading_factors(p, q, r)
    u0, s0, vt0 = np.linalg.svd(p @ q)
    np.testing.assert_allclose(s, s0[:r], rtol=1e-10)
    np.testing.assert_allclose(u * s @ vt, u0[:, :r] * s0[:r] @ vt0[:r], atol=1e-9 * s0[0])
    np.testing.assert_allclose(u.T @ u, np.eye(r), atol=1e-10)
    u, s, vt = lowrank.leading_factors(p, q, n + 3)
    assert s.shape == (n + 3,) and not s[n:].any() and not u[:, n:].any() and not vt[n:].any()
    np.testing.assert_allclose(u * s @ vt, p @ q, atol=1e-9 * s0[0])
