"""Low-rank compensation built from the expert weights alone (host-side weight preparation).

"KAIST drops calibration from MoE decoding ...", section "A reader built from weights
alone": the channels the sketch leaves out are compensated by a low-rank map derived from
the model's weights, with no calibration data.  The pages give no construction; the one
built here is the rank-r truncation of the least-squares linear predictor of what the
skipped channels would have added,

    M_e = argmin_M  E_x || y_skip(x) - M x ||^2,
    y_skip(x) = sum over the channels j the top-k selection leaves out of
                h_j(x) down[:, j],   h_j = silu(gate_j . x) * (up_j . x),

under the input prior x ~ N(0, I) (the only assumption in place of data).  With that prior
E[x x^T] = I and M_e = E[y_skip(x) x^T].  Channel j's share depends on x (up to the sketch
and the other channels' scores) only through a = gate_j . x and b = up_j . x, and the rest
of x is independent of them, so its column block lies in span(gate_j, up_j):

    E[h_j 1_skip x^T] = c_a gate_j^T + c_b up_j^T,
    [c_a, c_b] = C_j^-1 [E[h_j 1_skip a], E[h_j 1_skip b]],  C_j = Gram(gate_j, up_j).

Only these two moments per channel are estimated (Monte Carlo over seeded Gaussian
samples), so the d x d map carries no d-dimensional sampling noise.  Its SVD gives
A_e = U_r diag(s_r)^1/2 and B_e = diag(s_r)^1/2 V_r^T, which the block's kernels consume in
place of any other rank-r factors (A_e (B_e x) is added to the expert); with I < d the
SVD is taken of an I x I core of the product (``leading_factors``), not of the d x d map.  Under a zero-mean
prior the SwiGLU output is close to a quadratic form in x, whose best linear predictor is
small: on the Qwen3-30B-A3B-shaped synthetic block the map removes 1.4-2 % of the sparse
block's error against the dense one.

The selection inside the estimate follows the block's own rule: the ternary sketch of the
gate rows comes from the packer (msb_ternary_rows: threshold 0.7 * mean |W|, scale = mean
|W| of the kept entries), the scores are alpha_j * |T_j . x| and the k highest are kept
(ties to the lower index) over the Monte Carlo samples.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _lib


def _f32(a) -> np.ndarray:
    """BF16 bits (uint16) or float arrays -> float32."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32)
    return a.astype(np.float32)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> BF16 bits, round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + 0x7FFF
    return ((u + r) >> 16).astype(np.uint16)


def _ternary(gate: np.ndarray):
    """Per-row ternary sketch of gate [I][d] (float32): T in {-1, 0, 1} (as float32) and
    alpha [I], computed by the packer itself (msb_ternary_rows), so the selection inside
    the estimate is the one the block's sketch makes."""
    w = np.ascontiguousarray(gate, dtype=np.float32)
    rows, d = w.shape
    t = np.empty((rows, d), np.int8)
    alpha = np.empty(rows, np.float32)
    rc = _lib.load().msb_ternary_rows(w.ctypes.data_as(ctypes.c_void_p), rows, d,
                                      t.ctypes.data_as(ctypes.c_void_p),
                                      alpha.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("msb_ternary_rows: status %d" % rc)
    return t.astype(np.float32), alpha


def channel_moments(gate, up, down, k: int, x: np.ndarray, sketch=None):
    """Per channel j, the sample moments E[h_j 1_skip,j a_j] and E[h_j 1_skip,j b_j] with
    a_j = gate_j . x, b_j = up_j . x, h_j = silu(a_j) b_j and 1_skip,j the event that the
    top-k selection leaves j out.  sketch: the gate rows' (T, alpha) if already computed.
    Returns two [I] float64 arrays."""
    g_w, u_w = _f32(gate), _f32(up)
    t, alpha = _ternary(g_w) if sketch is None else sketch
    x = np.asarray(x, dtype=np.float32)
    scores = np.abs(x @ t.T) * alpha
    order = np.argsort(-scores, axis=1, kind="stable")
    skip = np.ones_like(scores, dtype=bool)
    np.put_along_axis(skip, order[:, :k], False, axis=1)
    a = (x @ g_w.T).astype(np.float64)
    b = (x @ u_w.T).astype(np.float64)
    h = a / (1.0 + np.exp(-a)) * b * skip
    return (h * a).mean(axis=0), (h * b).mean(axis=0)


def structured_rows(gate, up, ma: np.ndarray, mb: np.ndarray) -> np.ndarray:
    """Row j of the map's right factor, c_a,j gate_j + c_b,j up_j, from the channel
    moments (ma, mb) via the 2 x 2 Gram solve ([I][d], float64); a channel with collinear
    gate and up rows contributes nothing."""
    g_w = _f32(gate).astype(np.float64)
    u_w = _f32(up).astype(np.float64)
    gg, gu, uu = (g_w * g_w).sum(1), (g_w * u_w).sum(1), (u_w * u_w).sum(1)
    det = gg * uu - gu * gu
    ok = det > 1e-12 * np.maximum(gg * uu, 1e-300)
    ca = np.where(ok, (uu * ma - gu * mb) / np.where(ok, det, 1.0), 0.0)
    cb = np.where(ok, (gg * mb - gu * ma) / np.where(ok, det, 1.0), 0.0)
    return ca[:, None] * g_w + cb[:, None] * u_w


def structured_map(gate, up, down, ma: np.ndarray, mb: np.ndarray) -> np.ndarray:
    """M = sum_j down_j (c_a,j gate_j + c_b,j up_j)^T from the channel moments ([d][d])."""
    return _f32(down).astype(np.float64) @ structured_rows(gate, up, ma, mb)


def leading_factors(p: np.ndarray, q: np.ndarray, rank: int):
    """The leading `rank` singular triplets (U_r, s_r, V_r^T) of the product p @ q
    (p [d][n], q [n][d]).  With n < d the d x d product is not formed: from the QR
    factors p = Q_p R_p and q^T = Q_q R_q, p q = Q_p (R_p R_q^T) Q_q^T, so the SVD of the
    n x n core gives the same triplets.  Missing triplets (rank > min(d, n)) are zero."""
    d, n = p.shape
    if n >= d:
        u, s, vt = np.linalg.svd(p @ q)
    else:
        qp, rp = np.linalg.qr(p)
        qq, rq = np.linalg.qr(q.T)
        uc, s, vct = np.linalg.svd(rp @ rq.T)
        u, vt = qp @ uc, vct @ qq.T
    m = min(rank, s.size)
    ur, sr, vr = np.zeros((d, rank)), np.zeros(rank), np.zeros((rank, q.shape[1]))
    ur[:, :m], sr[:m], vr[:m] = u[:, :m], s[:m], vt[:m]
    return ur, sr, vr


def derive_lowrank(gate, up, down, k: int, rank: int, samples: int = 4096, seed: int = 0,
                   chunk: int = 512):
    """Rank-r compensation factors of every expert.

    gate, up: [E][I][d]; down: [E][d][I] (BF16 bits or floats); k: channels kept per
    (token, expert); rank: r.  Returns (lr_a [E][d][r], lr_b [E][r][d]) as BF16 bits, the
    layout the packer and the kernels take (see the module docstring for the map)."""
    gate, up, down = np.asarray(gate), np.asarray(up), np.asarray(down)
    e_n, inter, d = gate.shape
    lr_a = np.zeros((e_n, d, rank), np.uint16)
    lr_b = np.zeros((e_n, rank, d), np.uint16)
    if rank == 0:
        return lr_a, lr_b
    for e in range(e_n):
        rng = np.random.default_rng([seed, e])
        sketch = _ternary(_f32(gate[e]))
        ma, mb = np.zeros(inter), np.zeros(inter)
        done = 0
        while done < samples:
            n = min(chunk, samples - done)
            x = rng.standard_normal((n, d), dtype=np.float32)
            pa, pb = channel_moments(gate[e], up[e], down[e], k, x, sketch)
            ma += pa * n
            mb += pb * n
            done += n
        rows = structured_rows(gate[e], up[e], ma / samples, mb / samples)
        u, s, vt = leading_factors(_f32(down[e]).astype(np.float64), rows, rank)
        root = np.sqrt(s)  # balanced split: a zero map gives zero factors
        lr_a[e] = _bf16_bits(u * root + 0.0)  # + 0.0: no negative zeros
        lr_b[e] = _bf16_bits(root[:, None] * vt + 0.0)
    return lr_a, lr_b
