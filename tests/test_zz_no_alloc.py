"""The allocation-free batch-1 entry point, checked against the workspace entry point
and against the oracle.

Callers that own no device allocator (a plugin handed only its input and output
buffers, or code where a cudaMalloc is not permitted) use moe_sparse_block_noalloc;
its scratch is a static device array inside the library, shared by every call in the
process, so this file is collected last: the array then already holds what the other
tests' calls left in it, and the checks below show that each call starts clean anyway.
The file also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from parity import (OUT_RTOL, compare, device_layer, from_bf16_tensor, require_gpu,
                    to_bf16_tensor)

pytestmark = pytest.mark.gpu


def call_noalloc(lib, x, layer, k, out, trace=None):
    import torch
    cd = layer.dims.c()
    tr = trace.c() if trace is not None else None
    ptr = lambda t: None if t is None else t.data_ptr()
    return lib.moe_sparse_block_noalloc(
        x.data_ptr(), layer.router_t.data_ptr(), layer.records.data_ptr(), ptr(layer.sketch),
        ptr(layer.alpha), k, ptr(layer.lr_a), ptr(layer.lr_b), out.data_ptr(), ctypes.byref(cd),
        ctypes.byref(tr) if tr is not None else None, torch.cuda.current_stream().cuda_stream)


def traced(tr, out):
    return {"y": oracle.bf16_to_f64(from_bf16_tensor(out)), "ids": tr.expert_ids.cpu().numpy(),
            "w": tr.expert_w.cpu().numpy(), "sel": tr.sel.cpu().numpy().view(np.uint16),
            "sel_count": tr.sel_count.cpu().numpy(), "union": tr.union_count.cpu().numpy(),
            "scores": tr.scores.cpu().numpy() if tr.scores is not None else None}


@pytest.mark.parametrize("workload", [synth.TINY, synth.QWEN30B_BLOCK])
def test_noalloc_matches_workspace_entry_point(workload):
    msb = require_gpu()
    import torch
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    w = workload
    dev = device_layer(w)
    x = to_bf16_tensor(synth.activations(w, 17))
    ref = msb.moe_sparse_block(x, dev, w.k)           # existing entry point (with a workspace)
    torch.cuda.synchronize()
    ref64 = oracle.bf16_to_f64(from_bf16_tensor(ref))[0]
    lay = oracle.SynthLayer(w)
    for call in range(2):                              # two calls in a row share the scratch
        out = torch.empty_like(x)
        tr = msb.Trace(dev.dims, 1, w.k, scores=True)
        rc = call_noalloc(lib, x, dev, w.k, out, tr)
        assert rc == _lib.MSB_OK, lib.msb_strerror(rc)
        torch.cuda.synchronize()
        assert lib.msb_noalloc_check(torch.cuda.current_stream().cuda_stream) == _lib.MSB_OK
        g = traced(tr, out)
        rel = np.linalg.norm(g["y"][0] - ref64) / np.linalg.norm(ref64)
        assert rel <= OUT_RTOL, (call, rel)
        st = compare(synth.activations(w, 17), g, lay, w.top_e, w.k)   # routing, selection, output
        print(call, rel, st)


@pytest.mark.parametrize("k,rank", [(512, 0), (92, 0), (512, 16)])
def test_noalloc_dense_and_rank0(k, rank):
    """The dense path (k = I: no sketch read) and the block without compensation (rank 0:
    no A_e, B_e) through the allocation-free entry point, against the oracle."""
    msb = require_gpu()
    import torch
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    w = synth.TINY
    dev = device_layer(w, rank=rank)
    lay = oracle.SynthLayer(w)
    xb = synth.activations(w, 23)
    x = to_bf16_tensor(xb)
    out = torch.empty_like(x)
    tr = msb.Trace(dev.dims, 1, k, scores=True)
    rc = call_noalloc(lib, x, dev, k, out, tr)
    assert rc == _lib.MSB_OK, lib.msb_strerror(rc)
    torch.cuda.synchronize()
    assert lib.msb_noalloc_check(torch.cuda.current_stream().cuda_stream) == _lib.MSB_OK
    mode = "dense" if (k == w.inter and rank == 0) else "topk"
    compare(xb, traced(tr, out), lay, w.top_e, k, rank=rank, mode=mode,
            check_scores=(k != w.inter))


def test_noalloc_nonfinite_input_is_reported_then_recovers():
    """A NaN in x makes the router's logits NaN: msb_noalloc_check reports
    MSB_ENONFINITE for that call, and the next call is exact again."""
    msb = require_gpu()
    import torch
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    w = synth.QWEN30B_BLOCK
    dev = device_layer(w)
    stream = torch.cuda.current_stream().cuda_stream
    xb = synth.activations(w, 9)
    bad = xb.copy()
    bad[0, 17] = 0x7FC0  # bf16 quiet NaN
    out = torch.empty((1, w.d), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(lib, to_bf16_tensor(bad), dev, w.k, out) == _lib.MSB_OK
    assert lib.msb_noalloc_check(stream) == _lib.MSB_ENONFINITE
    assert lib.msb_noalloc_check(stream) == _lib.MSB_OK      # read and cleared
    tr = msb.Trace(dev.dims, 1, w.k, scores=True)
    assert call_noalloc(lib, to_bf16_tensor(xb), dev, w.k, out, tr) == _lib.MSB_OK
    assert lib.msb_noalloc_check(stream) == _lib.MSB_OK
    compare(xb, traced(tr, out), oracle.SynthLayer(w), w.top_e, w.k)


def test_noalloc_rejects_sizes_beyond_its_limit():
    require_gpu()
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    fake = 1 << 20  # never dereferenced: the size check fails first
    big = _lib.MsbDims(8256, 768, 128, 8, 32, 1)  # d above the 8192 limit
    rc = lib.moe_sparse_block_noalloc(fake, fake, fake, fake, fake, 138, fake, fake, fake * 2,
                                      ctypes.byref(big), None, None)
    assert rc == _lib.MSB_EUNSUPPORTED


def test_noalloc_at_its_size_limit():
    """d = MSB_NOALLOC_MAX_D = 8192: the static accumulator is used whole."""
    msb = require_gpu()
    import torch
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    w = synth.TINY.with_(name="wide_d8192_I512_E16_top4_k92_r16", d=8192, inter=512, experts=16,
                         top_e=4, k=92, rank=16, seed=0x7E57 + 40)
    dev = device_layer(w)
    xb = synth.activations(w, 8)
    x = to_bf16_tensor(xb)
    out = torch.empty_like(x)
    tr = msb.Trace(dev.dims, 1, w.k, scores=True)
    assert call_noalloc(lib, x, dev, w.k, out, tr) == _lib.MSB_OK
    torch.cuda.synchronize()
    assert lib.msb_noalloc_check(torch.cuda.current_stream().cuda_stream) == _lib.MSB_OK
    compare(xb, traced(tr, out), oracle.SynthLayer(w), w.top_e, w.k)
