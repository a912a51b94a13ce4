"""Offline preparation: every sparse-MoE layer of a safetensors checkpoint -> packed-layer
files (one per layer), so that a decoding process only uploads them.

    python -m token_top_expert_b200.prepare --out DIR --top-e 8 [--rank R --k K]
        [--records bf16|q4] [--layers 0,1,...] [--no-renorm] SHARD.safetensors ...

With --rank > 0 the compensation factors are derived from the weights for the channel
budget --k (``lowrank.derive_lowrank``).  Files are named layer_NNN.msbpack and carry
the checkpoint's shard names, the layer index and k in their metadata.
"""
from __future__ import annotations

import argparse
import os
import sys
import time

from . import checkpoint, packfile


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(prog="python -m token_top_expert_b200.prepare",
                                 description=__doc__.split("\n\n")[0])
    ap.add_argument("shards", nargs="+", help=".safetensors files of the checkpoint")
    ap.add_argument("--out", required=True, help="directory for the packed-layer files")
    ap.add_argument("--top-e", type=int, required=True, help="routed experts per token (trained)")
    ap.add_argument("--rank", type=int, default=0, help="compensation rank r (0: none)")
    ap.add_argument("--k", type=int, default=None, help="channel budget the factors compensate")
    ap.add_argument("--records", default="bf16", choices=["bf16", "q4"])
    ap.add_argument("--layers", default=None, help="comma-separated layer indices (default: all MoE layers)")
    ap.add_argument("--prefix", default="model.layers")
    ap.add_argument("--no-renorm", action="store_true", help="do not renormalise the top-K router weights")
    ap.add_argument("--lowrank-samples", type=int, default=4096)
    args = ap.parse_args(argv)
    if args.rank > 0 and args.k is None:
        ap.error("--rank > 0 needs --k")
    shards = checkpoint.Shards(args.shards)
    layers = (checkpoint.moe_layers(shards, args.prefix) if args.layers is None
              else [int(v) for v in args.layers.split(",") if v.strip()])
    if not layers:
        ap.error("no sparse-MoE layer found (prefix %r)" % args.prefix)
    os.makedirs(args.out, exist_ok=True)
    names = [os.path.basename(p) for p in args.shards]
    for layer in layers:
        t0 = time.time()
        dims, packed, lr_a, lr_b = checkpoint.pack_layer(
            shards, layer, args.top_e, rank=args.rank, k=args.k, renorm=0 if args.no_renorm else 1,
            records=args.records, prefix=args.prefix, lowrank_samples=args.lowrank_samples)
        path = os.path.join(args.out, "layer_%03d.msbpack" % layer)
        packfile.save(path, dims, packed, lr_a, lr_b, records=args.records,
                      meta={"shards": names, "layer": layer, "k": args.k})
        print("layer %d: d=%d I=%d E=%d -> %s (%.1f s)"
              % (layer, dims.d, dims.inter, dims.experts, path, time.time() - t0), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
