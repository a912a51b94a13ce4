"""GPU parity of the block on 4-bit channel records (moe_sparse_block_q4) against the
oracle over the dequantised layer (oracle.q4.Q4Layer): routing, scores from the sketch of
the dequantised gate rows, exact top-k, and the output, on the single-launch kernel at
batch 1 and at small batches, top-k and dense, with and without the low-rank term.
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import q4 as oq4
from parity import compare, from_bf16_tensor, require_gpu, to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msb():
    return require_gpu()


def q4_device_layer(msb, w, rank=None):
    r = w.rank if rank is None else rank
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, r, 1)
    pk = msb.pack_q4(lw.gate, lw.up, lw.down, lw.router, dims)
    dev = msb.PackedLayer.from_host(dims, pk, lw.lr_a, lw.lr_b)
    assert dev.q4
    return dev


def run_q4(msb, x_bits, dev, k, union=False):
    import torch
    B = x_bits.shape[0]
    tr = msb.Trace(dev.dims, B, k, scores=True, union=union)
    ws = msb.Workspace(dev.dims, B)
    out = msb.moe_sparse_block(to_bf16_tensor(x_bits), dev, k, workspace=ws, trace=tr)
    torch.cuda.synchronize()
    ws.check()
    return {"y": oracle.bf16_to_f64(from_bf16_tensor(out)), "ids": tr.expert_ids.cpu().numpy(),
            "w": tr.expert_w.cpu().numpy(), "sel": tr.sel.cpu().numpy().view(np.uint16),
            "sel_count": tr.sel_count.cpu().numpy(),
            "union": tr.union_count.cpu().numpy() if union else None,
            "scores": tr.scores.cpu().numpy()}


@pytest.mark.parametrize("workload,batch", [("qwen", 1), ("qwen", 4), ("tiny", 1), ("tiny", 3), ("large", 1)])
def test_q4_block_matches_oracle(msb, workload, batch):
    w = {"qwen": synth.QWEN30B_BLOCK, "tiny": synth.TINY, "large": synth.LARGE_BLOCK}[workload]
    dev = q4_device_layer(msb, w)
    assert msb.path_info(dev.dims, batch, w.k)["path"] == "single_launch"
    lay = oq4.Q4Layer(oracle.SynthLayer(w))
    x = synth.activations(w, 71, batch=batch)
    g = run_q4(msb, x, dev, w.k, union=(batch == 1))
    assert (g["sel_count"] == w.k).all()
    print(workload, batch, compare(x, g, lay, w.top_e, w.k))


@pytest.mark.parametrize("rank", [0, 16])
def test_q4_dense_and_rank(msb, rank):
    """k = I (every channel, no sketch read) and the low-rank term on and off."""
    w = synth.TINY
    dev = q4_device_layer(msb, w, rank=rank)
    lay = oq4.Q4Layer(oracle.SynthLayer(w))
    x = synth.activations(w, 72)
    for k in (w.inter, w.k):
        g = run_q4(msb, x, dev, k, union=True)
        mode = "dense" if (k == w.inter and rank == 0) else "topk"
        compare(x, g, lay, w.top_e, k, rank=rank, mode=mode, check_scores=(k != w.inter))


def test_q4_reads_fewer_bytes(msb):
    """The record the kernels gather: 3 d / 2 + 12 d / 64 bytes, rounded up to 16."""
    for d in (256, 2048, 4096):
        dims = msb.Dims(d, 512, 8, 2, 0, 1)
        assert msb.q4_record_bytes(dims) == oq4.record_bytes(d)


def test_q4_rejects_the_multi_kernel_path(msb):
    import torch
    from token_top_expert_b200 import MsbError
    w = synth.TINY
    dev = q4_device_layer(msb, w)
    x = to_bf16_tensor(synth.activations(w, 73, batch=32))   # above the single launch's 16 tokens
    with pytest.raises(MsbError):
        msb.moe_sparse_block(x, dev, w.k)
    torch.cuda.synchronize()
