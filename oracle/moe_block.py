"""FP64 restatement of one sparse-MoE block decode step (test infrastructure only).

Per token t the block does, in this order ([KAIST-EN] "A reader built from
weights alone" and "Top-k instead of a threshold"; tags are defined in the
package docstring):

1. route: logits = x . W_router, softmax over E, keep the top-K experts.
2. for each routed expert e:
   a. score every intermediate channel j with the ternary sketch of W_gate:
      s_j = alpha_j * |T_j . x|                                (sketch step)
   b. keep exactly the k highest-scoring channels              (top-k step)
   c. read only those channels' gate/up rows and down column, apply SwiGLU:
      y_e = sum_{j in S} silu(gate_j . x) * (up_j . x) * down[:, j]
   d. add the rank-r compensation of the skipped channels: y_e += A_e (B_e x)
3. combine: y = sum_e w_e * y_e

Arithmetic is FP64 throughout.  BF16 inputs are widened exactly.
"""
from __future__ import annotations

import math

import numpy as np

import synth


# ----------------------------------------------------------------------------- numbers

def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of BF16 bit patterns as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_to_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest BF16 value (ties to even), as float64.

    BF16 keeps 8 significant bits: v = m * 2**e with m in [0.5, 1); the result
    is round_half_even(m * 256) / 256 * 2**e.  (Normal range only: subnormal
    and overflowing values do not occur in the workloads.)
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


# ----------------------------------------------------------------------------- router

def route(x: np.ndarray, w_router: np.ndarray, top_e: int, renorm: bool):
    """Router of one token: softmax over x . W_router, then the top-K experts.

    The pages state that each token loads "the weights of the routed experts"
    ([KAIST-EN] opening paragraph); [TOPK-OVR] "Ce que ca fait" gives the shape
    (top 8 of 128 experts).  Readings: ranking uses the logits (the softmax is
    monotone), ties go to the lower expert index; with ``renorm`` the K kept
    probabilities are rescaled to sum to one.

    x: [d] float64, w_router: [d][E] float64.
    Returns (ids [K] in rank order, weights [K], logits [E]).
    """
    logits = x @ w_router
    p = np.exp(logits - logits.max())
    p = p / p.sum()
    order = np.lexsort((np.arange(logits.size), -logits))   # logit desc, index asc
    ids = order[:top_e]
    w = p[ids]
    if renorm:
        w = w / w.sum()
    return ids, w, logits


# ----------------------------------------------------------------------------- sketch

def ternary_sketch(w_rows: np.ndarray):
    """Ternary sketch of weight rows ([KAIST-EN] "A reader built from weights alone":
    channels are filtered with a ternary sketch of the weights; formula per [TWN]).

    For each row W (length d):
      delta = 0.7 * mean_i |W_i|
      T_i   = sign(W_i) if |W_i| > delta (strictly) else 0
      alpha = mean of |W_i| over {i : T_i != 0}, rounded to float32; 0 if none kept.

    The strict comparison |W_i| > 0.7 * (sum |W|) / d is evaluated as
    10 * d * |W_i| > 7 * sum|W|.  For BF16 rows both sides are exact in float64
    (the sum of up to 8192 BF16 magnitudes spanning less than 2**33 is exact),
    so an entry equal to delta is never kept.

    w_rows: [n][d] float64 (BF16 values).  Returns (T [n][d] int8, alpha [n] float32).
    """
    a = np.abs(w_rows)
    d = w_rows.shape[1]
    total = a.sum(axis=1)
    keep = (10.0 * d) * a > 7.0 * total[:, None]
    t = (np.sign(w_rows) * keep).astype(np.int8)
    n_kept = keep.sum(axis=1)
    kept_sum = (a * keep).sum(axis=1)
    alpha = np.where(n_kept > 0, kept_sum / np.maximum(n_kept, 1), 0.0).astype(np.float32)
    return t, alpha


def channel_scores(t: np.ndarray, alpha: np.ndarray, x: np.ndarray) -> np.ndarray:
    """Channel scores of one (token, expert): s_j = alpha_j * |T_j . x| (float64)."""
    return alpha.astype(np.float64) * np.abs(t.astype(np.float64) @ x)


# ----------------------------------------------------------------------------- selection

def topk_channels(s: np.ndarray, k: int) -> np.ndarray:
    """Exactly the k highest-scoring channels, ascending.

    [KAIST-EN] "Top-k instead of a threshold": per token keep the k channels
    with the highest scores, so the read budget is known in advance.  Ties:
    the lower channel index wins (key = (score desc, index asc)).
    """
    order = np.lexsort((np.arange(s.size), -s))
    return np.sort(order[:k])


def threshold_channels(s: np.ndarray, tau: float) -> np.ndarray:
    """The calibrated-threshold selector the pages compare against: {j : s_j > tau}
    ([KAIST-EN] "The threshold promises a budget but does not keep it")."""
    return np.nonzero(s > tau)[0]


def calibrate_threshold(scores: np.ndarray, budget: float) -> float:
    """Offline threshold for a read budget: the score above which a fraction
    ``budget`` of the pooled calibration scores lie.

    Sorted descending, tau is the (m+1)-th largest score with m = floor(N * budget),
    so exactly m calibration scores exceed it when there are no ties.
    """
    s = np.sort(np.asarray(scores, dtype=np.float64).ravel())[::-1]
    m = int(math.floor(s.size * budget))
    return float(s[min(m, s.size - 1)])


# ----------------------------------------------------------------------------- expert

def expert_output(x, gate, up, down, sel) -> np.ndarray:
    """Gathered SwiGLU expert over the selected channels only.

    Reads gate row j, up row j and down column j for j in sel ([KAIST-EN]
    opening paragraph: the selector "reads only their weights"; [TOPK-OVR]
    "Ce que ca fait": the expert MLP is gated), and returns
      y_e = sum_{j in sel} silu(gate_j . x) * (up_j . x) * down[:, j],
    silu(g) = g / (1 + exp(-g)).
    gate, up: [I][d]; down: [d][I]; x: [d].
    """
    sel = np.asarray(sel, dtype=np.int64)
    g = gate[sel] @ x
    u = up[sel] @ x
    h = g / (1.0 + np.exp(-g)) * u
    return down[:, sel] @ h


def lowrank_term(x, a, b) -> np.ndarray:
    """Rank-r compensation of the skipped channels, A_e (B_e x)
    ([KAIST-EN] "A reader built from weights alone": skipped channels are
    compensated by a low-rank map).  a: [d][r], b: [r][d]."""
    if a.shape[1] == 0:
        return np.zeros(a.shape[0])
    return a @ (b @ x)


# ----------------------------------------------------------------------------- weights

def _as_f64(a):
    a = np.asarray(a)
    return bf16_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


class ArrayLayer:
    """Weights of one layer held as arrays in model layout: BF16 bits (uint16)
    or plain float64 values (hand-built examples)."""

    def __init__(self, gate, up, down, router, lr_a=None, lr_b=None):
        self._gate, self._up, self._down = gate, up, down
        self._router = router
        self._a, self._b = lr_a, lr_b
        self._cache = {}
        self._sk = {}

    def router(self):
        if "router" not in self._cache:
            self._cache["router"] = _as_f64(self._router)
        return self._cache["router"]

    def expert(self, e):
        if e not in self._cache:
            d = self._gate.shape[2]
            a = _as_f64(self._a[e]) if self._a is not None else np.zeros((d, 0))
            b = _as_f64(self._b[e]) if self._b is not None else np.zeros((0, d))
            self._cache[e] = (_as_f64(self._gate[e]), _as_f64(self._up[e]),
                              _as_f64(self._down[e]), a, b)
        return self._cache[e]

    def sketch(self, e):
        if e not in self._sk:
            self._sk[e] = ternary_sketch(self.expert(e)[0])
        return self._sk[e]


class SynthLayer(ArrayLayer):
    """Weights of one layer regenerated expert by expert from the seeded generator.
    At most ``max_cache`` experts' float64 weights are kept (least recently used
    are dropped and regenerated on demand); sketches are kept for every expert."""

    def __init__(self, workload, layer=0, max_cache=12):
        self.w, self.layer = workload, layer
        self._cache = {}
        self._sk = {}
        self._order = []
        self._max = max_cache

    def router(self):
        if "router" not in self._cache:
            self._cache["router"] = bf16_to_f64(synth.router(self.w, self.layer))
        return self._cache["router"]

    def expert(self, e):
        if e in self._order:
            self._order.remove(e)
        self._order.append(e)
        while len(self._order) > self._max:
            self._cache.pop(self._order.pop(0), None)
        if e not in self._cache:
            w, l = self.w, self.layer
            if w.rank:
                a = bf16_to_f64(synth.lowrank_a(w, e, l))
                b = bf16_to_f64(synth.lowrank_b(w, e, l))
            else:
                a, b = np.zeros((w.d, 0)), np.zeros((0, w.d))
            self._cache[e] = (bf16_to_f64(synth.expert_gate(w, e, l)),
                              bf16_to_f64(synth.expert_up(w, e, l)),
                              bf16_to_f64(synth.expert_down(w, e, l)), a, b)
        return self._cache[e]


# ----------------------------------------------------------------------------- block

def moe_block(x_bits, layer, top_e, k, renorm=True, rank=None, mode="topk", tau=None,
              forced_sel=None, forced_ids=None):
    """One sparse-MoE block decode step for a batch of tokens.

    x_bits: [B][d] BF16 bits (or float64 values).  layer: ArrayLayer/SynthLayer.
    mode: "topk" (k channels per (token, expert)), "threshold" ({s > tau}),
          or "dense" (every channel, no sketch).
    rank: use only the first ``rank`` columns/rows of A_e/B_e (None = all; 0 = none).
    forced_sel: optional {(t, e): channels} that replaces the selection of those
                pairs (used to re-drive the oracle with another selection when
                two channels are tied within the score epsilon).
    forced_ids: optional {t: expert ids} replacing the router's choice (logit ties).

    Returns a dict: y [B][d] float64, ids [B][K], w [B][K], logits [B][E],
    sel {(t, e): ascending channels}, scores {(t, e): s}, union {e: channels}.
    """
    x_all = np.asarray(x_bits)
    x_all = bf16_to_f64(x_all) if x_all.dtype == np.uint16 else x_all.astype(np.float64)
    B, d = x_all.shape
    w_router = layer.router()
    out = {"y": np.zeros((B, d)), "ids": [], "w": [], "logits": [], "sel": {}, "scores": {},
           "union": {}}
    for t in range(B):
        x = x_all[t]
        ids, w, logits = route(x, w_router, top_e, renorm)
        if forced_ids is not None and t in forced_ids:
            ids = np.asarray(forced_ids[t])
            p = np.exp(logits - logits.max())
            p = p / p.sum()
            w = p[ids] / (p[ids].sum() if renorm else 1.0)
        out["ids"].append(ids)
        out["w"].append(w)
        out["logits"].append(logits)
        y = np.zeros(d)
        for e, we in zip(ids, w):
            e = int(e)
            gate, up, down, a, b = layer.expert(e)
            if mode == "dense":
                sel = np.arange(gate.shape[0])
            else:
                tt, alpha = layer.sketch(e)
                s = channel_scores(tt, alpha, x)
                out["scores"][(t, e)] = s
                sel = topk_channels(s, k) if mode == "topk" else threshold_channels(s, tau)
            if forced_sel is not None and (t, e) in forced_sel:
                sel = np.asarray(forced_sel[(t, e)], dtype=np.int64)
            out["sel"][(t, e)] = sel
            ye = expert_output(x, gate, up, down, sel)
            r = 0 if mode == "dense" else (a.shape[1] if rank is None else rank)
            if r > 0:
                ye = ye + lowrank_term(x, a[:, :r], b[:r, :])
            y += we * ye
            prev = out["union"].get(e, np.zeros(0, dtype=np.int64))
            out["union"][e] = np.union1d(prev, sel)
        out["y"][t] = y
    out["ids"] = np.array(out["ids"])
    out["w"] = np.array(out["w"])
    out["logits"] = np.array(out["logits"])
    return out


def dense_moe(x_bits, layer, top_e, renorm=True):
    """The dense MoE block: every channel of every routed expert, no sketch, no low-rank."""
    return moe_block(x_bits, layer, top_e, k=None, renorm=renorm, mode="dense")


def read_bytes(union_sizes, d, inter, rank, dense=False) -> int:
    """Weight bytes one block step must read (the skipped channels are not read):
    per used expert, the sketch (2 bits per gate weight, I*d/4 bytes), the row
    scales (4I), the selected channels' gate row + up row + down column in BF16
    (6d per channel of the union over the step's tokens) and A_e, B_e (4dr).
    The dense path reads neither sketch, scales nor low-rank factors."""
    total = 0
    for u in union_sizes:
        total += 6 * d * int(u)
        if not dense:
            total += inter * d // 4 + 4 * inter + 4 * d * rank
    return total


# ----------------------------------------------------------------------------- stack glue

def rmsnorm(h, eps=1e-6) -> np.ndarray:
    """RMSNorm with unit weight: h / sqrt(mean(h**2) + eps), row-wise."""
    h = np.asarray(h, dtype=np.float64)
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def stack_layer(h, layer, top_e, k, renorm=True, mode="topk", x_override=None, eps=1e-6):
    """One pre-norm decode layer of the MoE stack (attention omitted):
    x = BF16(RMSNorm(h)); h_next = h + MoE(x).

    The MoE block takes BF16 activations, so the normalised state is rounded to
    BF16 at the block boundary.  ``x_override`` ([B][d] BF16 bits) replaces that
    input, so a layer can be checked on exactly the activations another
    implementation fed it.  Returns (h_next, x_bits_used_as_f64, block result).
    """
    h = np.asarray(h, dtype=np.float64)
    x = round_to_bf16(rmsnorm(h, eps)) if x_override is None else bf16_to_f64(x_override)
    res = moe_block(x, layer, top_e, k, renorm=renorm, mode=mode)
    return h + res["y"], x, res
