"""Helpers shared by the GPU parity tests: build device layers from the seeded
generator, run libmsb through its C ABI, and compare with the oracle.

Comparison rules (the stated tolerances):
  * router: the K expert ids match exactly, except where the oracle's logits of
    the swapped experts are within 1e-6 * max|logit| of each other (then the
    oracle is re-driven with the GPU's experts);
  * selection: the kept channel sets match exactly, except channels whose oracle
    scores lie within 1e-6 * s_(k) of the oracle's k-th score s_(k) (then the
    oracle is re-driven with the GPU's sets);
  * output: per token, ||y_gpu - y_oracle||_2 <= 2e-2 * ||y_oracle||_2 (BF16
    output, FP32 accumulation);
  * read volume: every (token, expert) keeps exactly k channels, and each
    expert's reported union size equals the size of the union of its kept sets.
"""
from __future__ import annotations

import functools

import numpy as np

import oracle
import synth

SCORE_EPS = 1e-6
LOGIT_EPS = 1e-6
OUT_RTOL = 2e-2


def require_gpu():
    import pytest
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_top_expert_b200 import build
    build.build()
    import token_top_expert_b200 as msb
    msb.load_library()
    return msb


@functools.lru_cache(maxsize=2)
def device_layer(w: synth.Workload, layer: int = 0, rank: int | None = None):
    import token_top_expert_b200 as msb
    r = w.rank if rank is None else rank
    lw = synth.layer_weights(w, layer)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, r, 1)
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    return msb.PackedLayer.from_host(dims, pk, lw.lr_a, lw.lr_b)


def to_bf16_tensor(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_bf16_tensor(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_gpu(x_bits, dev, k, general=False, threshold=None, scores=True):
    import token_top_expert_b200 as msb
    import torch
    B = x_bits.shape[0]
    x = to_bf16_tensor(x_bits)
    tr = msb.Trace(dev.dims, B, k, scores=scores, threshold=threshold is not None)
    ws = msb.Workspace(dev.dims, B)
    if threshold is None:
        out = msb.moe_sparse_block(x, dev, k, workspace=ws, trace=tr, general=general)
    else:
        out = msb.moe_sparse_block_threshold(x, dev, threshold, workspace=ws, trace=tr)
    torch.cuda.synchronize()
    ws.check()
    res = {
        "y": oracle.bf16_to_f64(from_bf16_tensor(out)),
        "ids": tr.expert_ids.cpu().numpy(),
        "w": tr.expert_w.cpu().numpy(),
        "sel": tr.sel.cpu().numpy().view(np.uint16),
        "sel_count": tr.sel_count.cpu().numpy(),
        "union": tr.union_count.cpu().numpy(),
        "scores": tr.scores.cpu().numpy() if tr.scores is not None else None,
    }
    return res


def compare(x_bits, g, lay, top_e, k, rank=None, mode="topk", tau=None, tokens=None,
            check_scores=True):
    """Check one GPU call `g` against the oracle on the tokens `tokens` (default all).
    Returns a stats dict.  Raises AssertionError on any violation."""
    B = x_bits.shape[0]
    tokens = range(B) if tokens is None else tokens
    stats = {"max_rel_l2": 0.0, "swaps": 0, "router_ties": 0, "max_score_rel": 0.0, "pairs": 0}
    inter = lay.expert(int(g["ids"][0][0]))[0].shape[0]
    for t in tokens:
        xt = x_bits[t:t + 1]
        ref = oracle.moe_block(xt, lay, top_e, k, rank=rank, mode=mode, tau=tau)
        gid = [int(v) for v in g["ids"][t]]
        oid = [int(v) for v in ref["ids"][0]]
        forced_ids = None
        if gid != oid:
            logits = ref["logits"][0]
            scale = LOGIT_EPS * np.abs(logits).max()
            for a, b in zip(gid, oid):
                assert abs(logits[a] - logits[b]) <= scale, ("router", t, gid, oid)
            forced_ids = {0: gid}
            stats["router_ties"] += 1
            ref = oracle.moe_block(xt, lay, top_e, k, rank=rank, mode=mode, tau=tau,
                                   forced_ids=forced_ids)
        np.testing.assert_allclose(g["w"][t], ref["w"][0], rtol=1e-5, atol=1e-7)
        forced = {}
        for r, e in enumerate(gid):
            stats["pairs"] += 1
            if mode == "dense":
                continue
            n = int(g["sel_count"][t][r])
            gs = np.sort(g["sel"][t][r][:n].astype(np.int64))
            assert np.all(np.diff(gs) > 0), "GPU selection not strictly ascending"
            if mode == "topk":
                assert n == k, ("read budget", t, e, n, k)
            s = ref["scores"][(0, e)]
            os_ = ref["sel"][(0, e)]
            if check_scores and g["scores"] is not None:
                gsc = g["scores"][t][r][:inter].astype(np.float64)
                denom = max(np.abs(s).max(), 1e-30)
                rel = np.abs(gsc - s).max() / denom
                stats["max_score_rel"] = max(stats["max_score_rel"], rel)
                assert rel < 1e-5, ("scores", t, e, rel)
            if set(gs.tolist()) != set(os_.tolist()):
                if mode == "topk":
                    sk = np.sort(s)[::-1][k - 1]
                    bound = SCORE_EPS * sk
                else:
                    sk = tau
                    bound = SCORE_EPS * abs(tau)
                for j in set(gs.tolist()) ^ set(os_.tolist()):
                    assert abs(s[j] - sk) <= bound, ("selection", t, e, j, s[j], sk)
                stats["swaps"] += 1
                forced[(0, e)] = gs
        if forced or forced_ids is not None:
            ref = oracle.moe_block(xt, lay, top_e, k, rank=rank, mode=mode, tau=tau,
                                   forced_sel=forced or None, forced_ids=forced_ids)
        yr = ref["y"][0]
        rel = np.linalg.norm(g["y"][t] - yr) / max(np.linalg.norm(yr), 1e-30)
        stats["max_rel_l2"] = max(stats["max_rel_l2"], rel)
        assert rel <= OUT_RTOL, ("output", t, rel)
    return stats


def check_union(g, top_e):
    """Each used expert's union size equals |union of its tokens' kept sets|."""
    B = g["ids"].shape[0]
    sets = {}
    for t in range(B):
        for r in range(top_e):
            e = int(g["ids"][t][r])
            n = int(g["sel_count"][t][r])
            sets.setdefault(e, set()).update(g["sel"][t][r][:n].tolist())
    for e in range(g["union"].shape[0]):
        assert int(g["union"][e]) == len(sets.get(e, ())), e
    return sum(len(v) for v in sets.values())
