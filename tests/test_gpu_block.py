"""GPU parity of the sparse-MoE block (libmsb through its C ABI) against the oracle.

Tolerances (stated in tests/parity.py): router ids and kept channel sets exact
up to 1e-6-relative ties, outputs within 2e-2 relative L2 per token, exactly k
channels per (token, expert).
"""
import numpy as np
import pytest

import oracle
import synth
from parity import check_union, compare, device_layer, require_gpu, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msb():
    return require_gpu()


def dev_from_arrays(msb, lw, w, rank):
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, rank, 1)
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    return msb.PackedLayer.from_host(dims, pk, lw.lr_a, lw.lr_b)


# ------------------------------------------------------------------ tiny block, every step

@pytest.mark.parametrize("general", [False, True])
def test_tiny_block_all_steps(msb, general):
    w = synth.TINY
    dev = device_layer(w)
    info = msb.path_info(dev.dims, 1, w.k, general=general)
    print(info)
    assert info["path"] == ("multi_kernel" if general else "single_launch")
    lay = oracle.SynthLayer(w, max_cache=w.experts)
    worst = 0.0
    for step in range(w.steps):
        x = synth.activations(w, step)
        g = run_gpu(x, dev, w.k, general=general)
        st = compare(x, g, lay, w.top_e, w.k)
        worst = max(worst, st["max_rel_l2"])
        assert check_union(g, w.top_e) == w.top_e * w.k
    print("tiny worst rel-L2 %.2e" % worst)


# ------------------------------------------------------------------ Qwen3-30B-A3B-shaped block

@pytest.mark.parametrize("general", [False, True])
def test_qwen_block_batch1(msb, general):
    w = synth.QWEN30B_BLOCK
    dev = device_layer(w)
    info = msb.path_info(dev.dims, 1, w.k, general=general)
    print(info)
    assert info["path"] == ("multi_kernel" if general else "single_launch")
    lay = oracle.SynthLayer(w)
    for step in (0, 1, 7, 123, 999):
        x = synth.activations(w, step)
        g = run_gpu(x, dev, w.k, general=general)
        st = compare(x, g, lay, w.top_e, w.k)
        assert check_union(g, w.top_e) == w.top_e * w.k
        print(step, st)


@pytest.mark.parametrize("general", [False, True])
def test_qwen_block_dense_k768(msb, general):
    w = synth.QWEN30B_BLOCK
    dev = device_layer(w, rank=0)
    assert msb.path_info(dev.dims, 1, w.inter, general=general)["path"] == (
        "multi_kernel" if general else "single_launch")
    lay = oracle.SynthLayer(w)
    for step in (0, 5):
        x = synth.activations(w, step)
        g = run_gpu(x, dev, w.inter, general=general)
        st = compare(x, g, lay, w.top_e, w.inter, mode="dense")
        used = set(int(e) for e in g["ids"][0])
        for e in range(w.experts):
            assert int(g["union"][e]) == (w.inter if e in used else 0)
        print(step, st)


@pytest.mark.parametrize("batch", [4, 16, 64])
def test_batch_budget_k100(msb, batch):
    w = synth.QWEN30B_BLOCK_13
    dev = device_layer(synth.QWEN30B_BLOCK)   # same block weights, 13% budget
    lay = oracle.SynthLayer(synth.QWEN30B_BLOCK)
    x = synth.activations(w, 0, batch=batch)
    g = run_gpu(x, dev, w.k)
    assert (g["sel_count"] == w.k).all()
    total = check_union(g, w.top_e)
    tokens = range(batch) if batch <= 4 else range(0, batch, max(1, batch // 6))
    st = compare(x, g, lay, w.top_e, w.k, tokens=tokens)
    print(batch, "union channels", total, st)
    # the batch path must give every token the same result as a batch-1 call
    for t in list(tokens)[:2]:
        g1 = run_gpu(x[t:t + 1], dev, w.k, general=True)
        assert (g1["ids"][0] == g["ids"][t]).all()
        assert np.array_equal(np.sort(g1["sel"][0], axis=1), np.sort(g["sel"][t], axis=1))
        rel = np.linalg.norm(g1["y"][0] - g["y"][t]) / np.linalg.norm(g1["y"][0])
        assert rel < 1e-2


def test_threshold_comparator(msb):
    w = synth.QWEN30B_BLOCK_13
    base = synth.QWEN30B_BLOCK
    dev = device_layer(base)
    lay = oracle.SynthLayer(base)
    # calibrate tau on held-out tokens with the oracle's scores
    calib = synth.calibration_activations(w, 0, 8)
    pooled = []
    for t in range(calib.shape[0]):
        ref = oracle.moe_block(calib[t:t + 1], lay, w.top_e, w.k)
        pooled.extend(s for s in ref["scores"].values())
    tau = oracle.calibrate_threshold(np.concatenate(pooled), w.k / w.inter)
    x = synth.activations(w, 3, batch=4)
    g = run_gpu(x, dev, w.k, threshold=tau)
    st = compare(x, g, lay, w.top_e, w.k, mode="threshold", tau=tau)
    counts = g["sel_count"].ravel()
    check_union(g, w.top_e)
    print("threshold tau %.4g read fraction mean %.4f std %.4f min %d max %d" %
          (tau, counts.mean() / w.inter, counts.std() / w.inter, counts.min(), counts.max()), st)


# ------------------------------------------------------------------ large-expert block

@pytest.mark.parametrize("batch", [1, 8])
def test_large_block(msb, batch):
    w = synth.LARGE_BLOCK
    dev = device_layer(w)
    if batch == 1:
        assert msb.path_info(dev.dims, 1, w.k)["path"] == "single_launch"
    lay = oracle.SynthLayer(w)
    x = synth.activations(w, 11, batch=batch)
    g = run_gpu(x, dev, w.k)
    assert (g["sel_count"] == w.k).all()
    check_union(g, w.top_e)
    st = compare(x, g, lay, w.top_e, w.k, tokens=range(min(batch, 3)))
    print(batch, st)


# ------------------------------------------------------------------ edge cases

EDGE = [
    # d, I, E, K, k, r, batch
    (64, 33, 4, 2, 1, 0, 1),
    (64, 33, 4, 2, 32, 1, 3),
    (64, 33, 4, 4, 33, 0, 1),        # k = I (dense), K = E
    (256, 512, 8, 2, 511, 1, 1),
    (256, 512, 8, 2, 1, 16, 64),
    (256, 512, 1, 1, 92, 16, 3),     # a single expert
    (128, 48, 16, 16, 7, 2, 5),      # every expert routed
]


@pytest.mark.parametrize("d,inter,E,K,k,r,batch", EDGE)
@pytest.mark.parametrize("general", [False, True])
def test_edge_shapes(msb, d, inter, E, K, k, r, batch, general):
    w = synth.TINY.with_(d=d, inter=inter, experts=E, top_e=K, k=k, rank=r, seed=1000 + d + inter)
    lw = synth.layer_weights(w)
    dev = dev_from_arrays(msb, lw, w, r)
    lay = oracle.ArrayLayer(lw.gate, lw.up, lw.down, lw.router, lw.lr_a, lw.lr_b)
    x = synth.activations(w, 0, batch=batch)
    g = run_gpu(x, dev, k, general=general)
    mode = "topk"
    if k == inter and r == 0:
        mode = "dense"
    st = compare(x, g, lay, K, k, rank=r, mode=mode)
    if mode == "topk":
        check_union(g, K)
    print(st)


def test_zero_rows_and_duplicate_scores(msb):
    """All-zero gate rows score exactly 0 and tie; duplicated rows tie exactly;
    the lower channel index must win in both cases."""
    w = synth.TINY.with_(d=256, inter=64, experts=2, top_e=2, k=40, rank=0, seed=77)
    lw = synth.layer_weights(w)
    for e in range(2):
        lw.gate[e, 0::2] = 0            # 32 zero rows -> alpha = 0, score 0
        lw.gate[e, 3] = lw.gate[e, 5]   # duplicated rows -> identical scores
        lw.gate[e, 7] = lw.gate[e, 5]
    dev = dev_from_arrays(msb, lw, w, 0)
    lay = oracle.ArrayLayer(lw.gate, lw.up, lw.down, lw.router)
    for step in range(4):
        x = synth.activations(w, step)
        g = run_gpu(x, dev, w.k)
        compare(x, g, lay, 2, w.k, rank=0)
        # 32 nonzero rows + the 8 lowest-index zero rows
        for r in range(2):
            sel = set(g["sel"][0][r].tolist())
            assert {0, 2, 4, 6, 8, 10, 12, 14} <= sel
            assert not ({16, 18, 20} & sel)


@pytest.mark.parametrize("general", [False, True])
def test_nonfinite_input_is_flagged_then_recovers(msb, general):
    """A NaN in x makes every router logit NaN: the call is flagged (msb_check
    returns MSB_ENONFINITE, the output is undefined) and the next call on the same
    workspace is exact again (accumulators and counters were restored)."""
    import torch
    import token_top_expert_b200 as m
    from parity import to_bf16_tensor
    w = synth.QWEN30B_BLOCK
    dev = device_layer(w)
    ws = m.Workspace(dev.dims, 1)
    x = synth.activations(w, 9)
    bad = x.copy()
    bad[0, 17] = 0x7FC0  # bf16 quiet NaN
    m.moe_sparse_block(to_bf16_tensor(bad), dev, w.k, workspace=ws, general=general)
    torch.cuda.synchronize()
    with pytest.raises(m.MsbError) as exc:
        ws.check()
    assert exc.value.status == -5
    tr = m.Trace(dev.dims, 1, w.k, scores=True)
    out = m.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, trace=tr, general=general)
    torch.cuda.synchronize()
    ws.check()
    from parity import from_bf16_tensor
    g = {"y": oracle.bf16_to_f64(from_bf16_tensor(out)), "ids": tr.expert_ids.cpu().numpy(),
         "w": tr.expert_w.cpu().numpy(), "sel": tr.sel.cpu().numpy().view(np.uint16),
         "sel_count": tr.sel_count.cpu().numpy(), "union": tr.union_count.cpu().numpy(),
         "scores": tr.scores.cpu().numpy()}
    compare(x, g, oracle.SynthLayer(w), w.top_e, w.k)


@pytest.mark.parametrize("top_e,batch", [(4, 1), (6, 1), (4, 4), (6, 16)])
def test_expert_count_override(msb, top_e, batch):
    """Routing to fewer experts than trained ("MoE top_k override (--moe-top-k)"),
    combined with the channel top-k: the oracle with K = top_e."""
    import torch
    import token_top_expert_b200 as m
    from parity import from_bf16_tensor, to_bf16_tensor
    w = synth.QWEN30B_BLOCK
    dev = device_layer(w)
    lay = oracle.SynthLayer(w)
    dims_k = m.Dims(w.d, w.inter, w.experts, top_e, w.rank, 1)
    x = synth.activations(w, 21, batch=batch)
    tr = m.Trace(dims_k, batch, w.k, scores=True)
    ws = m.Workspace(dev.dims, batch)
    out = m.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, trace=tr, top_e=top_e)
    torch.cuda.synchronize()
    ws.check()
    if batch == 1:
        assert msb.path_info(dims_k, 1, w.k)["path"] == "single_launch"
    g = {"y": oracle.bf16_to_f64(from_bf16_tensor(out)), "ids": tr.expert_ids.cpu().numpy(),
         "w": tr.expert_w.cpu().numpy(), "sel": tr.sel.cpu().numpy().view(np.uint16),
         "sel_count": tr.sel_count.cpu().numpy(), "union": tr.union_count.cpu().numpy(),
         "scores": tr.scores.cpu().numpy()}
    compare(x, g, lay, top_e, w.k)
    assert (g["union"] > 0).sum() <= top_e * batch
    with pytest.raises(m.MsbError):
        m.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, top_e=w.top_e + 1)


@pytest.mark.parametrize("batch", [1, 4])
def test_weight_derived_lowrank(msb, batch):
    """The block with compensation factors derived from the weights alone (in place of
    seeded ones): same kernels, same parity bar, against the oracle given the same factors."""
    from token_top_expert_b200 import lowrank
    w = synth.TINY
    lw = synth.layer_weights(w)
    a, b = lowrank.derive_lowrank(lw.gate, lw.up, lw.down, k=w.k, rank=w.rank, samples=1024)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, w.rank, 1)
    dev = msb.PackedLayer.from_host(dims, msb.pack(lw.gate, lw.up, lw.down, lw.router, dims), a, b)
    lay = oracle.ArrayLayer(lw.gate, lw.up, lw.down, lw.router, a, b)
    for step in range(3):
        x = synth.activations(w, 300 + step, batch=batch)
        g = run_gpu(x, dev, w.k)
        compare(x, g, lay, w.top_e, w.k, rank=w.rank)


def test_selection_is_deterministic(msb):
    w = synth.QWEN30B_BLOCK
    dev = device_layer(w)
    x = synth.activations(w, 42)
    a = run_gpu(x, dev, w.k)
    b = run_gpu(x, dev, w.k)
    c = run_gpu(x, dev, w.k, general=True)
    assert np.array_equal(a["ids"], b["ids"]) and np.array_equal(a["sel"], b["sel"])
    assert np.array_equal(a["ids"], c["ids"]) and np.array_equal(a["sel"], c["sel"])
    assert np.array_equal(a["scores"], b["scores"])


def test_workspace_reuse_across_batch_sizes(msb):
    import torch
    import token_top_expert_b200 as m
    from parity import from_bf16_tensor, to_bf16_tensor
    w = synth.TINY
    dev = device_layer(w)
    ws = m.Workspace(dev.dims, 16)
    outs = {}
    for B, general in ((16, True), (1, False), (3, True), (1, True), (1, False)):
        x = synth.activations(w, 5, batch=16)[:B]
        y = m.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, general=general)
        torch.cuda.synchronize()
        outs.setdefault(B, []).append(oracle.bf16_to_f64(from_bf16_tensor(y)))
    ws.check()
    for B, ys in outs.items():
        for y in ys[1:]:
            assert np.linalg.norm(y - ys[0]) <= 1e-2 * np.linalg.norm(ys[0])
    assert np.linalg.norm(outs[1][0][0] - outs[16][0][0]) <= 1e-2 * np.linalg.norm(outs[1][0][0])


# ------------------------------------------------------------------ small batches, one launch

@pytest.mark.parametrize("workload,batch", [("qwen13", 2), ("qwen13", 4), ("qwen13", 16), ("tiny", 3)])
def test_small_batch_single_launch(msb, workload, batch):
    """Batches of up to 16 tokens on the single-launch kernel (one cluster per (token,
    routed expert) pair; asked for, since 16 tokens at d = 2048 default to the
    multi-kernel path): every token against the oracle; consecutive calls share the
    workspace's accumulator and slice counters."""
    import torch
    from parity import from_bf16_tensor, to_bf16_tensor
    w = synth.QWEN30B_BLOCK_13 if workload == "qwen13" else synth.TINY
    dev = device_layer(w)
    assert msb.path_info(dev.dims, batch, w.k, single=True)["path"] == "single_launch"
    lay = oracle.SynthLayer(w)
    ws = msb.Workspace(dev.dims, batch)
    for step in range(2):
        x = synth.activations(w, 60 + step, batch=batch)
        tr = msb.Trace(dev.dims, batch, w.k, scores=True, union=False)
        out = msb.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, trace=tr, single=True)
        torch.cuda.synchronize()
        ws.check()
        g = {"y": oracle.bf16_to_f64(from_bf16_tensor(out)), "ids": tr.expert_ids.cpu().numpy(),
             "w": tr.expert_w.cpu().numpy(), "sel": tr.sel.cpu().numpy().view(np.uint16),
             "sel_count": tr.sel_count.cpu().numpy(), "union": None,
             "scores": tr.scores.cpu().numpy()}
        assert (g["sel_count"] == w.k).all()
        print(batch, step, compare(x, g, lay, w.top_e, w.k))


@pytest.mark.parametrize("workload,batch,path", [
    ("qwen13", 12, "single_launch"), ("qwen13", 16, "multi_kernel"),
    ("large", 3, "single_launch"), ("large", 4, "multi_kernel"), ("wide", 1, "single_launch"),
    ("wide", 2, "multi_kernel"), ("tiny", 16, "single_launch")])
def test_default_path_follows_the_crossover(msb, workload, batch, path):
    """The default path: the single launch up to 12 (2048 / d)^2 tokens (1..16), the
    multi-kernel path above; MSB_FLAG_SINGLE keeps the single launch up to 16 tokens."""
    # the shapes of the workloads the parity tests run (d, I, E, K, r) and their k
    shape, k = {"qwen13": ((2048, 768, 128, 8, 32), 100), "large": ((4096, 1536, 128, 8, 64), 276),
                "wide": ((8192, 512, 16, 4, 16), 92), "tiny": ((256, 512, 8, 2, 16), 92)}[workload]
    dims = msb.Dims(*shape, 1)
    assert msb.path_info(dims, batch, k)["path"] == path
    assert msb.path_info(dims, batch, k, single=True)["path"] == "single_launch"
    assert msb.path_info(dims, batch, k, general=True, single=True)["path"] == "multi_kernel"
