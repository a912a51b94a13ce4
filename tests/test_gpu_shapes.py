"""GPU parity at the edges of the accepted shapes: the large block at the batch sizes the
benchmark runs (32, 128), the largest batch (256) and the largest hidden size (d = 8192)
on both paths.  Batches are checked on sampled tokens (first, middle, last): the oracle
runs one token at a time in FP64.
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


def _sampled(batch):
    return sorted({0, batch // 2, batch - 1})


@pytest.mark.parametrize("batch", [32, 128])
def test_large_block_batches(msb, batch):
    w = synth.LARGE_BLOCK
    dev = device_layer(w)
    lay = oracle.SynthLayer(w)
    x = synth.activations(w, 13, batch=batch)
    g = run_gpu(x, dev, w.k)
    assert (g["sel_count"] == w.k).all()
    check_union(g, w.top_e)
    print(batch, compare(x, g, lay, w.top_e, w.k, tokens=_sampled(batch)))


def test_largest_batch(msb):
    w = synth.QWEN30B_BLOCK_13
    dev = device_layer(w)
    lay = oracle.SynthLayer(w)
    x = synth.activations(w, 5, batch=256)
    g = run_gpu(x, dev, w.k)
    assert (g["sel_count"] == w.k).all()
    check_union(g, w.top_e)
    print(compare(x, g, lay, w.top_e, w.k, tokens=_sampled(256)))


# the largest hidden size the ABI accepts; a small expert set keeps the weights at
# E * I * 3 * d * 2 bytes = 16 * 512 * 3 * 8192 * 2 = 402 MB
WIDE = synth.TINY.with_(name="wide_d8192_I512_E16_top4_k92_r16", d=8192, inter=512, experts=16,
                        top_e=4, k=92, rank=16, seed=0x7E57 + 40)


@pytest.mark.parametrize("batch,general", [(1, False), (1, True), (3, False)])
def test_widest_hidden_size(msb, batch, general):
    w = WIDE
    dev = device_layer(w)
    path = msb.path_info(dev.dims, batch, w.k, general=general)["path"]
    print(path)
    if batch == 1 and not general:
        assert path == "single_launch"
    lay = oracle.SynthLayer(w)
    x = synth.activations(w, 3, batch=batch)
    g = run_gpu(x, dev, w.k, general=general)
    assert (g["sel_count"] == w.k).all()
    check_union(g, w.top_e)
    print(batch, general, compare(x, g, lay, w.top_e, w.k))


@pytest.mark.parametrize("rank", [8, 12, 128])
def test_low_rank_term_ranks(msb, rank):
    """A_e z on the multi-kernel path for ranks whose rows of A_e are 16-byte multiples
    (staged through shared memory: 8, and 128, the largest accepted) and one that is not
    (12: read from registers)."""
    w = synth.TINY.with_(name="tiny_r%d" % rank, rank=rank)
    dev = device_layer(w)
    assert msb.path_info(dev.dims, 24, w.k)["path"] != "single_launch"
    lay = oracle.SynthLayer(w)
    x = synth.activations(w, 19, batch=24)
    g = run_gpu(x, dev, w.k)
    assert (g["sel_count"] == w.k).all()
    print(rank, compare(x, g, lay, w.top_e, w.k, rank=rank, tokens=_sampled(24)))
