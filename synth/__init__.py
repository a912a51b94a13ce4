"""Seeded synthetic inputs for the sparse-MoE block decode workloads.

This module only draws numbers: Gaussian BF16 weight matrices, the activations
x, and the choice of heavy-tailed rows.  It holds none of the block's
arithmetic (no router, sketch, selection or expert math), so both the CPU
oracle and the GPU path can take their inputs from it.

Every tensor is a pure function of (workload seed, layer, tensor id, index):
each piece is drawn from its own numpy ``Generator(Philox(SeedSequence(...)))``
stream, so one expert (or one decode step) can be regenerated without drawing
the rest.  Values are N(0, sigma) drawn in float32 and rounded once to BF16
(round to nearest, ties to even); BF16 tensors are returned as their uint16
bit patterns.

Weight shapes follow the usual model layout:
  gate[e], up[e]  : [I][d]   (row j = channel j)
  down[e]         : [d][I]   (column j = channel j)
  router          : [d][E]
  lowrank A[e]    : [d][r]
  lowrank B[e]    : [r][d]
  x[step]         : [batch][d]
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# tensor ids (part of every stream key)
T_GATE, T_UP, T_DOWN, T_ROUTER, T_LR_A, T_LR_B, T_X, T_HEAVY, T_CALIB_X, T_H0 = range(1, 11)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and value distribution of one MoE-block workload."""
    name: str
    d: int              # hidden size
    inter: int          # expert intermediate size I
    experts: int        # E
    top_e: int          # routed experts per token
    k: int              # channels kept per (token, expert)
    rank: int           # low-rank compensation rank r
    sigma: float        # std of the expert / router / low-rank weights
    heavy_frac: float   # fraction of channels whose gate/up rows are scaled
    heavy_scale: float  # the scale applied to those rows
    batch: int          # tokens per decode step
    steps: int          # decode steps (fresh x each step)
    seed: int
    layers: int = 1     # >1 only for the stacked decode workload

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def budget_k(budget: float, inter: int) -> int:
    """Channels kept for a read budget given as a fraction of I (nearest integer)."""
    return int(round(budget * inter))


# The workloads.  Seeds are 0x7E57 + workload index.
TINY = Workload("tiny_d256_I512_E8_top2_k92_r16", d=256, inter=512, experts=8, top_e=2, k=92,
                rank=16, sigma=0.02, heavy_frac=0.0, heavy_scale=1.0, batch=1, steps=64,
                seed=0x7E57 + 0)
QWEN30B_BLOCK = Workload("qwen3_30b_a3b_block_d2048_I768_E128_top8_k138_r32", d=2048, inter=768,
                         experts=128, top_e=8, k=138, rank=32, sigma=0.02, heavy_frac=0.05,
                         heavy_scale=4.0, batch=1, steps=1000, seed=0x7E57 + 1)
QWEN30B_BLOCK_13 = QWEN30B_BLOCK.with_(name="qwen3_30b_a3b_block_k100_batch", k=100,
                                       seed=0x7E57 + 2)
LARGE_BLOCK = Workload("large_block_d4096_I1536_E128_top8_k276_r64", d=4096, inter=1536,
                       experts=128, top_e=8, k=276, rank=64, sigma=0.015, heavy_frac=0.05,
                       heavy_scale=4.0, batch=1, steps=500, seed=0x7E57 + 3)
STACK48 = QWEN30B_BLOCK.with_(name="stack48_qwen3_30b_a3b_block", layers=48, steps=256,
                              seed=0x7E57 + 4)

WORKLOADS = {w.name: w for w in (TINY, QWEN30B_BLOCK, QWEN30B_BLOCK_13, LARGE_BLOCK, STACK48)}


def _gen(w: Workload, layer: int, tid: int, index: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([w.seed, layer, tid, index])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(g: np.random.Generator, shape, sigma: float) -> np.ndarray:
    z = g.standard_normal(int(np.prod(shape)), dtype=np.float32) * np.float32(sigma)
    return f32_to_bf16_bits(z).reshape(shape)


def heavy_rows(w: Workload, e: int, layer: int = 0) -> np.ndarray:
    """Sorted channel indices of expert e whose gate/up rows are scaled."""
    n = int(round(w.heavy_frac * w.inter))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    g = _gen(w, layer, T_HEAVY, e)
    return np.sort(g.choice(w.inter, size=n, replace=False))


def _scaled_rows_bf16(w: Workload, e: int, layer: int, tid: int) -> np.ndarray:
    g = _gen(w, layer, tid, e)
    z = g.standard_normal(w.inter * w.d, dtype=np.float32).reshape(w.inter, w.d) * np.float32(w.sigma)
    rows = heavy_rows(w, e, layer)
    if rows.size:
        z[rows] *= np.float32(w.heavy_scale)
    return f32_to_bf16_bits(z)


def expert_gate(w: Workload, e: int, layer: int = 0) -> np.ndarray:
    """W_gate of expert e, [I][d] BF16 bits."""
    return _scaled_rows_bf16(w, e, layer, T_GATE)


def expert_up(w: Workload, e: int, layer: int = 0) -> np.ndarray:
    """W_up of expert e, [I][d] BF16 bits."""
    return _scaled_rows_bf16(w, e, layer, T_UP)


def expert_down(w: Workload, e: int, layer: int = 0) -> np.ndarray:
    """W_down of expert e, [d][I] BF16 bits."""
    return _normal_bf16(_gen(w, layer, T_DOWN, e), (w.d, w.inter), w.sigma)


def router(w: Workload, layer: int = 0) -> np.ndarray:
    """W_router, [d][E] BF16 bits."""
    return _normal_bf16(_gen(w, layer, T_ROUTER, 0), (w.d, w.experts), w.sigma)


def lowrank_a(w: Workload, e: int, layer: int = 0) -> np.ndarray:
    """A_e, [d][r] BF16 bits."""
    return _normal_bf16(_gen(w, layer, T_LR_A, e), (w.d, w.rank), w.sigma)


def lowrank_b(w: Workload, e: int, layer: int = 0) -> np.ndarray:
    """B_e, [r][d] BF16 bits."""
    return _normal_bf16(_gen(w, layer, T_LR_B, e), (w.rank, w.d), w.sigma)


def activations(w: Workload, step: int, batch: int | None = None, tid: int = T_X) -> np.ndarray:
    """x for one decode step, [batch][d] BF16 bits, N(0, 1)."""
    b = w.batch if batch is None else batch
    return _normal_bf16(_gen(w, 0, tid, step), (b, w.d), 1.0)


def calibration_activations(w: Workload, index: int, batch: int) -> np.ndarray:
    """Held-out tokens for threshold calibration (streams disjoint from activations())."""
    return activations(w, index, batch, tid=T_CALIB_X)


def stack_initial_hidden(w: Workload, step: int, batch: int | None = None) -> np.ndarray:
    """Residual-stream input h of layer 0 for one decode step, [batch][d] float32, N(0, 1)."""
    b = w.batch if batch is None else batch
    return _gen(w, 0, T_H0, step).standard_normal(b * w.d, dtype=np.float32).reshape(b, w.d)


@dataclasses.dataclass
class LayerWeights:
    """All weights of one MoE layer as BF16 bit arrays (model layout)."""
    gate: np.ndarray    # [E][I][d]
    up: np.ndarray      # [E][I][d]
    down: np.ndarray    # [E][d][I]
    router: np.ndarray  # [d][E]
    lr_a: np.ndarray    # [E][d][r]
    lr_b: np.ndarray    # [E][r][d]


def layer_weights(w: Workload, layer: int = 0, threads: int = 8) -> LayerWeights:
    """Every expert of one layer (threaded: each expert is an independent stream)."""
    E, I, d, r = w.experts, w.inter, w.d, w.rank
    gate = np.empty((E, I, d), np.uint16)
    up = np.empty((E, I, d), np.uint16)
    down = np.empty((E, d, I), np.uint16)
    lr_a = np.empty((E, d, r), np.uint16)
    lr_b = np.empty((E, r, d), np.uint16)

    def one(e):
        gate[e] = expert_gate(w, e, layer)
        up[e] = expert_up(w, e, layer)
        down[e] = expert_down(w, e, layer)
        if r:
            lr_a[e] = lowrank_a(w, e, layer)
            lr_b[e] = lowrank_b(w, e, layer)

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(one, range(E)))
    return LayerWeights(gate, up, down, router(w, layer), lr_a, lr_b)
