"""The allocation-free batch-1 entry point, checked against the workspace entry point.

Callers that own no device allocator (a plugin handed only its input and output
buffers, or code where a cudaMalloc is not permitted) use moe_sparse_block_noalloc;
its scratch is a static device array inside the library.  This file runs last
(pytest collects files in name order) so a failure here never hides the others.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from parity import OUT_RTOL, device_layer, from_bf16_tensor, require_gpu, to_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("workload", [synth.TINY, synth.QWEN30B_BLOCK])
def test_noalloc_matches_workspace_entry_point(workload):
    msb = require_gpu()
    import torch
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    w = workload
    dev = device_layer(w)
    msb_layer = dev
    x = to_bf16_tensor(synth.activations(w, 17))
    ref = msb.moe_sparse_block(x, dev, w.k)           # existing entry point (with a workspace)
    torch.cuda.synchronize()
    ref64 = oracle.bf16_to_f64(from_bf16_tensor(ref))[0]
    cd = dev.dims.c()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):                              # two calls in a row share the scratch
        out = torch.empty_like(x)
        rc = lib.moe_sparse_block_noalloc(
            x.data_ptr(), msb_layer.router_t.data_ptr(), msb_layer.records.data_ptr(),
            msb_layer.sketch.data_ptr(), msb_layer.alpha.data_ptr(), w.k,
            msb_layer.lr_a.data_ptr(), msb_layer.lr_b.data_ptr(), out.data_ptr(),
            ctypes.byref(cd), None, stream)
        assert rc == _lib.MSB_OK, lib.msb_strerror(rc)
        torch.cuda.synchronize()
        y = oracle.bf16_to_f64(from_bf16_tensor(out))[0]
        rel = np.linalg.norm(y - ref64) / np.linalg.norm(ref64)
        assert rel <= OUT_RTOL, (call, rel)


def test_noalloc_rejects_sizes_beyond_its_limit():
    require_gpu()
    from token_top_expert_b200 import _lib
    lib = _lib.load()
    fake = 1 << 20  # never dereferenced: the size check fails first
    big = _lib.MsbDims(8256, 768, 128, 8, 32, 1)  # d above the 8192 limit
    rc = lib.moe_sparse_block_noalloc(fake, fake, fake, fake, fake, 138, fake, fake, fake * 2,
                                      ctypes.byref(big), None, None)
    assert rc == _lib.MSB_EUNSUPPORTED
