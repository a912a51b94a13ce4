"""Run by tests/test_gpu_wait_expiry.py in a process of its own: against the instrumented
build (libmsb_instr.so), make one bounded wait run out on purpose and check that the call
is flagged and that the next call on the same workspace matches the oracle again.

For each path (the single-launch kernel, then the multi-kernel gather) the library is
told to withhold one bulk copy (never issued, so no fault: the wait for it simply runs
out) with a 50 us wait limit.  Prints one JSON line with each path's msb_check status of
the sabotaged call, the status of the next call and its parity statistics.
"""
import json
import os
import sys

os.environ["MSB_VARIANT"] = "instr"
HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402
from token_top_expert_b200 import build  # noqa: E402

build.build(variant="instr")
import token_top_expert_b200 as msb  # noqa: E402
from token_top_expert_b200 import _lib  # noqa: E402
from parity import compare, from_bf16_tensor, to_bf16_tensor  # noqa: E402

WAIT_NS = 50_000


def main():
    assert _lib.LIB_PATH.endswith("libmsb_instr.so")
    lib = _lib.load()
    torch.cuda.set_device(0)
    w = synth.QWEN30B_BLOCK.with_(experts=16, seed=0x7E57 + 1)
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, w.rank, 1)
    dev = msb.PackedLayer.from_host(dims, msb.pack(lw.gate, lw.up, lw.down, lw.router, dims),
                                    lw.lr_a, lw.lr_b)
    lay = oracle.ArrayLayer(lw.gate, lw.up, lw.down, lw.router, lw.lr_a, lw.lr_b)
    res = {}
    for general, skip in ((False, 1), (True, 2)):
        ws = msb.Workspace(dims, 1)
        x = synth.activations(w, 31 + skip)
        assert lib.msb_debug_inject(skip, WAIT_NS) == 0
        path = msb.path_info(dims, 1, w.k, general=general)["path"]
        msb.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, general=general)
        torch.cuda.synchronize()
        bad = lib.msb_check(ws.ptr, torch.cuda.current_stream().cuda_stream)
        assert lib.msb_debug_inject(0, 0) == 0
        tr = msb.Trace(dims, 1, w.k, scores=True)
        out = msb.moe_sparse_block(to_bf16_tensor(x), dev, w.k, workspace=ws, trace=tr,
                                   general=general)
        torch.cuda.synchronize()
        good = lib.msb_check(ws.ptr, torch.cuda.current_stream().cuda_stream)
        g = {"y": oracle.bf16_to_f64(from_bf16_tensor(out)), "ids": tr.expert_ids.cpu().numpy(),
             "w": tr.expert_w.cpu().numpy(), "sel": tr.sel.cpu().numpy().view(np.uint16),
             "sel_count": tr.sel_count.cpu().numpy(), "union": tr.union_count.cpu().numpy(),
             "scores": tr.scores.cpu().numpy()}
        st = compare(x, g, lay, w.top_e, w.k)
        res["general" if general else "single_launch"] = {
            "path": path, "sabotaged_status": int(bad), "next_status": int(good),
            "next_max_rel_l2": float(st["max_rel_l2"])}
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
