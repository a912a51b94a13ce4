"""4-bit channel records: FP64 restatement (test infrastructure only).

[TOPK-OVR] "Combinaison avec d'autres optimisations": the expert-count override is
measured on 4-bit (and 3-bit) quantised checkpoints of the same model, so the gathered
channels may be held at 4 bits instead of BF16.  The page names the checkpoints but not
their format.  Reading taken (group-wise affine, the usual form of such checkpoints):

  every run of G = 64 consecutive weights of a gate row, an up row or a down column has
  a BF16 scale s and a BF16 bias b, every weight a code q in {0, ..., 15}, and the weight
  the block computes with is s * q + b.

Quantising one group w_0 .. w_{G-1} (BF16 values):

  b   = bf16(min_i w_i)                       (exact for BF16 inputs)
  s   = bf16((max_i w_i - min_i w_i) / 15)    (round to nearest even)
  q_i = clamp(round_half_even((w_i - b) / s), 0, 15),   q_i = 0 when s = 0.

Down columns are grouped along d (not along I), so that one channel's gate row, up row
and down column stay one self-contained record.  The block over 4-bit records is the
block over the dequantised weights: the sketch is the ternary sketch of the dequantised
gate rows, and scores, top-k, SwiGLU, low-rank and combine are unchanged
(``oracle.moe_block`` on a ``Q4Layer``).
"""
from __future__ import annotations

import numpy as np

from .moe_block import ArrayLayer, round_to_bf16

GROUP = 64


def quantize_groups(w, group: int = GROUP):
    """Group-wise affine 4-bit codes of the last axis of ``w`` (float64 BF16 values).

    Returns (q uint8 [..., n], s [..., n/group], b [..., n/group]), s and b as
    float64 values of BF16 numbers.
    """
    w = np.asarray(w, dtype=np.float64)
    n = w.shape[-1]
    assert n % group == 0
    g = w.reshape(w.shape[:-1] + (n // group, group))
    lo, hi = g.min(axis=-1), g.max(axis=-1)
    b = round_to_bf16(lo)
    s = round_to_bf16((hi - lo) / 15.0)
    safe = np.where(s > 0, s, 1.0)
    t = np.where(s[..., None] > 0, (g - b[..., None]) / safe[..., None], 0.0)
    q = np.clip(np.rint(t), 0, 15).astype(np.uint8)   # np.rint: half to even
    return q.reshape(w.shape), s, b


def dequantize_groups(q, s, b, group: int = GROUP) -> np.ndarray:
    """Weights s * q + b of group-wise 4-bit codes (float64)."""
    q = np.asarray(q, dtype=np.float64)
    n = q.shape[-1]
    g = q.reshape(q.shape[:-1] + (n // group, group))
    return (s[..., None] * g + b[..., None]).reshape(q.shape)


def q4_weights(gate, up, down, group: int = GROUP):
    """The weights of one expert as its 4-bit records hold them.

    gate, up: [I][d] (rows quantised along d); down: [d][I] (each column j quantised
    along d).  Returns the dequantised (gate, up, down) in the same layouts."""
    qg = dequantize_groups(*quantize_groups(gate, group), group)
    qu = dequantize_groups(*quantize_groups(up, group), group)
    qd = dequantize_groups(*quantize_groups(np.asarray(down).T, group), group).T
    return qg, qu, np.ascontiguousarray(qd)


class Q4Layer(ArrayLayer):
    """A layer whose experts are read from 4-bit channel records: wraps another layer
    (ArrayLayer or SynthLayer) and serves its experts' dequantised weights; router and
    low-rank factors are those of the wrapped layer (they stay BF16).  At most
    ``max_cache`` experts' dequantised weights are kept (least recently used are
    dropped and rebuilt on demand); sketches are kept for every expert."""

    def __init__(self, base, group: int = GROUP, max_cache: int = 12):
        self.base, self.group = base, group
        self._cache = {}
        self._sk = {}
        self._order = []
        self._max = max_cache

    def router(self):
        return self.base.router()

    def expert(self, e):
        if e in self._order:
            self._order.remove(e)
        self._order.append(e)
        while len(self._order) > self._max:
            self._cache.pop(self._order.pop(0), None)
        if e not in self._cache:
            gate, up, down, a, b = self.base.expert(e)
            self._cache[e] = q4_weights(gate, up, down, self.group) + (a, b)
        return self._cache[e]


def record_bytes(d: int, group: int = GROUP) -> int:
    """Bytes of one 4-bit channel record: 3d codes at 4 bits, then a BF16 scale and
    bias per group of the three vectors, padded to a multiple of 16 bytes."""
    raw = 3 * d // 2 + 3 * (d // group) * 4
    return (raw + 15) // 16 * 16


def read_bytes(union_sizes, d, inter, rank, group: int = GROUP) -> int:
    """Weight bytes one block step reads with 4-bit records: as the BF16 block
    (sketch I*d/4, row scales 4I, low-rank 4dr per used expert) with each selected
    channel costing one 4-bit record instead of 6d bytes."""
    rec = record_bytes(d, group)
    return sum(rec * int(u) + inter * d // 4 + 4 * inter + 4 * d * rank for u in union_sizes)
