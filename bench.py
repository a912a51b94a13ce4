"""Benchmark: MoE-block decode tokens/s and achieved HBM bandwidth at batch 1, 18% budget.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--k K] [--batch B] [--rank R]

Workload (default): the Qwen3-30B-A3B-shaped block, d=2048, I=768, E=128, top-8,
k=138 (18%), r=32, batch 1, BF16 weights N(0, 0.02) with 5% of channels x4,
x ~ N(0, 1); 1000 decode steps with fresh seeded x per step (synthetic data).

One step = one call of the whole block (router, sketch scoring, top-k,
gathered SwiGLU + down, low-rank term, combine) on one batch.  The K timed
steps run as replays of a CUDA graph that holds the 1000-step decode
sequence; consecutive steps read different weight replicas (R copies of the
packed layer, R * 1.3 GB >> 126 MB L2), so every step reads its bytes from HBM.

Printed JSON (rank 0, one line): value = tokens/s over all ranks, e2e = the
same through the public Python/C-ABI call with pinned host x/out copies per
step, roofline = the step's algorithmic bytes / device time vs the measured
HBM copy bandwidth, cpu_baseline = the FP64 CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# the sources the single-launch kernel is built from (its recorded traffic stays valid
# while these are unchanged)
FUSED_SOURCES = ("token_top_expert_b200/csrc/fused.cu", "token_top_expert_b200/csrc/fused.h",
                 "token_top_expert_b200/csrc/common.cuh", "token_top_expert_b200/csrc/block_scan.cuh",
                 "include/msb.h")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in FUSED_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    r = rec.get(kernel, {}).get(workload)
    if not r or r.get("source_hash") != kernel_source_hash():
        return None
    return r.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica_throughput(ms_local: float, units_per_rank: float, dist=None, device=None):
    """Whole-job throughput of independent replicas (one per rank): the job takes the
    slowest rank's device time (max over ranks) and processes every rank's units.
    Returns (ms, units per second over all ranks).  Every rank takes the same
    collective steps."""
    import torch
    ms, world = ms_local, 1
    if dist is not None and dist.is_available() and dist.is_initialized():
        t = torch.tensor([ms_local], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        world = dist.get_world_size()
    return ms, units_per_rank * world / (ms / 1e3)


def block_launches(path, dense, rank):
    """Kernels one block call launches: the single-launch kernel, or the multi-kernel
    path's router, score (not for a dense block without compensation), select (not
    dense), union, gather and finalize."""
    if path == "single_launch":
        return 1
    return 4 + (1 if (not dense or rank > 0) else 0) + (0 if dense else 1)


def q4_record_bytes(d):
    """One 4-bit channel record: 3d codes at 4 bits, a BF16 scale and bias per group of 64
    of the three vectors, padded to 16 bytes."""
    return (3 * d // 2 + 3 * (d // 64) * 4 + 15) // 16 * 16


def algorithmic_bytes(w, k, rank, union_sizes, dense, q4=False):
    """Bytes the method must read for one step: per used expert the sketch
    (I*d/4), row scales (4I), the union of selected channel records (6d each, or the
    4-bit record size) and A_e, B_e (4dr).  The dense path (k = I) reads no sketch or
    scales; it still adds the low-rank term when rank > 0."""
    rec = q4_record_bytes(w.d) if q4 else 6 * w.d
    total = 0
    for u in union_sizes:
        if u == 0:
            continue
        total += rec * int(u) + 4 * w.d * rank
        if not dense:
            total += w.inter * w.d // 4 + 4 * w.inter
    return total


def oracle_sample(w, k, rank, xs, budget_s=15.0, max_tokens=None, top_e=None, timed_s=12.0, q4=False):
    """Time the FP64 CPU oracle, as it stands, on the first tokens of the step
    sequence: a warm pass (bounded by budget_s) fills its weight caches, then passes
    over the same tokens are timed until at least timed_s seconds of oracle work.
    Returns (tokens/s, tokens, seconds, threads)."""
    import oracle
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        threads = max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:  # noqa: BLE001
        threads = 1
    lay = oracle.SynthLayer(w, max_cache=w.experts)
    if q4:
        from oracle import q4 as oq4
        lay = oq4.Q4Layer(lay, max_cache=w.experts)
    toks = []
    t0 = time.time()
    n = 0
    while n < len(xs) and (max_tokens is None or n < max_tokens):
        oracle.moe_block(xs[n], lay, top_e or w.top_e, k, rank=rank)   # warm: generate + sketch
        toks.append(n)
        n += 1
        if time.time() - t0 > budget_s:
            break
    t1 = time.time()
    passes = 0
    while True:
        for i in toks:
            oracle.moe_block(xs[i], lay, top_e or w.top_e, k, rank=rank)
        passes += 1
        if time.time() - t1 >= timed_s:
            break
    dt = time.time() - t1
    ntok = passes * len(toks) * xs[0].shape[0]
    return ntok / dt, ntok, dt, threads


def run_reference(args, w, world, rank):
    """The reference arm: the CPU oracle timed on the same workload (bounded sample)."""
    if rank != 0:
        return
    xs = [synth.activations(w, s, batch=args.batch) for s in range(max(min(args.steps, 1000), 1))]
    budget = 60.0
    v, ntok, dt, threads = oracle_sample(w, args.k, args.rank, xs, top_e=args.top_e, budget_s=budget / 4,
                                         max_tokens=args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * args.batch / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": "%d token-blocks: passes over the first steps of the decode "
                                   "sequence (weights cached by an untimed pass), %.1f s" % (ntok, dt)},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


METRIC = "MoE-block decode tokens/s and achieved HBM GB/s vs peak at B=1, 18% budget"

# %globaltimer marks of the single-launch kernel (instrumented build), in kernel order
PHASE_MARKS = ("start", "x and router rows in", "logits in", "experts ranked", "sketch tiles in",
               "sketch scored", "scores and z pushed", "scores in", "top-k selected",
               "positions found", "records issued, A_e z done", "first record pair used",
               "records done", "partial outputs in", "end")


def run_phase_marks(args, w, local):
    """Per-phase timeline of the single-launch kernel from its instrumented build
    (libmsb_instr.so): `steps` launches captured back to back in one CUDA graph (weight
    replicas rotated, as in the timed bench), each CTA's %globaltimer at every phase
    boundary.  Times are relative to the moment the step's last CTA had x and its router
    rows (the end of the wait for the previous launch).  Prints one JSON line."""
    import torch
    import token_top_expert_b200 as msb
    from token_top_expert_b200 import _lib
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, args.rank, 1)
    pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
    base = msb.PackedLayer.from_host(dims, pk, lw.lr_a, lw.lr_b, device=dev)
    del lw, pk
    layers = [base] + [base.clone() for _ in range(args.replicas - 1)]
    plan = msb.path_info(dims, 1, args.k)
    if plan["path"] != "single_launch":
        raise SystemExit("phase marks need the single-launch path, got %s" % plan)
    n = max(8, min(args.steps, 400))
    grid = plan["cluster_size"] * w.top_e
    nseq = min(w.steps, 1000)
    xs = torch.from_numpy(np.stack([synth.activations(w, s) for s in range(nseq)]).view(np.int16)).to(dev).view(torch.bfloat16)
    outs = torch.empty_like(xs)
    ws = msb.Workspace(dims, 1, dev)
    marks = torch.zeros((n, grid, 16), dtype=torch.int64, device=dev)
    stream = torch.cuda.Stream(dev)
    lib = _lib.load()

    def launch(i, mk):
        lib.msb_debug_set_marks(mk)
        msb.moe_sparse_block(xs[i % nseq], layers[i % args.replicas], args.k, out=outs[i % nseq],
                             workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            launch(i, None)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(n):
            launch(i, marks[i].data_ptr())
    lib.msb_debug_set_marks(None)
    graph.replay()
    graph.replay()
    stream.synchronize()
    ws.check(stream)
    m = marks.cpu().numpy().astype(np.float64)
    t = m[:, :, :len(PHASE_MARKS)]
    t0 = t[:, :, 1].max(axis=1)[:, None, None]  # every CTA has x: the step's work starts
    rel = (t - t0) / 1e3  # us
    skip = min(4, n // 4)
    rel = rel[skip:]
    ends = t[skip:, :, len(PHASE_MARKS) - 1].max(axis=1)
    period = float(np.median(np.diff(ends))) / 1e3
    phases = []
    for i, name in enumerate(PHASE_MARKS):
        v = rel[:, :, i]
        phases.append({"mark": name, "median_us": round(float(np.median(v)), 3),
                       "max_us": round(float(np.median(v.max(axis=1))), 3)})
    smids = m[skip, :, 15].astype(int)
    per_sm = np.bincount(smids, minlength=148)
    line = {"metric": "single-launch kernel phase timeline (median over launches)",
            "workload": w.name, "k": args.k, "rank": args.rank, "launches": int(rel.shape[0]),
            "ctas": grid, "plan": plan, "period_us": round(period, 3),
            "sms_used": int((per_sm > 0).sum()), "sms_with_two_ctas": int((per_sm > 1).sum()),
            "phases": phases, "source_hash": kernel_source_hash(),
            "note": "times relative to the moment the step's last CTA had x and its router rows; "
                    "median = median over CTAs, max = slowest CTA (both medians over launches)"}
    print(json.dumps(line), flush=True)
    del graph


def config_of(w, args):
    return {"workload": w.name, "d": w.d, "I": w.inter, "E": w.experts,
            "top_e": args.top_e or w.top_e, "trained_top_e": w.top_e,
            "k": args.k, "budget": round(args.k / w.inter, 4), "rank": args.rank,
            "global_batch": args.batch * args.gpus, "batch_per_gpu": args.batch,
            "decode_steps": w.steps, "replicas": args.replicas,
            "l2": "inputs larger than L2: %d weight replicas rotated per step" % args.replicas,
            "parallelism": "replicas" if args.gpus > 1 else "single",
            "records": "4-bit (group 64, affine)" if getattr(args, "q4", False) else "bf16"}


def run_stack(args, w, world, rank, local):
    """Stacked decode: `layers` MoE blocks with per-layer seeded weights, pre-norm
    residual glue (h <- h + MoE_l(BF16(RMSNorm(h)))), attention omitted.  A step is
    one token (or batch) through every layer."""
    import torch
    import token_top_expert_b200 as msb
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L = w.layers
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, w.rank, 1)
    built = []
    t0 = time.time()
    for l in range(L):
        lw = synth.layer_weights(w, l)
        pk = msb.pack(lw.gate, lw.up, lw.down, lw.router, dims)
        built.append(msb.PackedLayer.from_host(dims, pk, lw.lr_a, lw.lr_b, device=dev))
        del lw, pk
    setup_s = time.time() - t0
    grid = [(args.k, args.batch)]
    if args.stack_grid:
        grid = [(k, b) for b in (1, 32) for k in (100, 138, w.inter)]
    for k, B in grid:
        r = 0 if k == w.inter else w.rank
        layers = built if r == w.rank else [lay.without_lowrank() for lay in built]
        run_stack_one(args, w, local, dev, layers, k, B, r, setup_s)


def run_stack_one(args, w, local, dev, layers, k, B, rank, setup_s):
    import torch
    import token_top_expert_b200 as msb
    L = w.layers
    dims = layers[0].dims
    nseq = 16
    h0 = torch.from_numpy(np.stack([synth.stack_initial_hidden(w, s, B) for s in range(nseq)])).to(dev)
    h = torch.empty((B, w.d), dtype=torch.float32, device=dev)
    xb = torch.empty((B, w.d), dtype=torch.bfloat16, device=dev)
    yb = torch.empty_like(xb)
    ws = msb.Workspace(dims, B, dev)
    stream = torch.cuda.Stream(dev)
    dense = k == w.inter

    def step(s, trace=None):
        h.copy_(h0[s % nseq])
        for l in range(L):
            msb.residual_rmsnorm(h, yb if l > 0 else None, xb, stream=stream)
            msb.moe_sparse_block(xb, layers[l], k, out=yb, workspace=ws, trace=trace,
                                 stream=stream)
        msb.residual_rmsnorm(h, yb, xb, stream=stream)

    # bytes of one step, from traced calls
    tr = msb.Trace(dims, B, k)
    byts = 0
    with torch.cuda.stream(stream):
        h.copy_(h0[0])
        for l in range(L):
            msb.residual_rmsnorm(h, yb if l > 0 else None, xb, stream=stream)
            msb.moe_sparse_block(xb, layers[l], k, out=yb, workspace=ws, trace=tr, stream=stream)
            stream.synchronize()
            byts += algorithmic_bytes(w, k, rank, tr.union_count.cpu().tolist(), dense)
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    ws.check(stream)
    G = min(nseq, args.steps)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            step(i)
    graph.replay()
    stream.synchronize()
    reps = max(1, args.steps // G)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                graph.replay()
            e1.record(stream)
        stream.synchronize()
    ms = e0.elapsed_time(e1)
    steps = reps * G
    ms_per_step = ms / steps
    peak, peak_kind = peaks()
    achieved = byts / (ms_per_step * 1e-3) / 1e9
    plan = msb.path_info(dims, B, k)
    line = {
        "metric": "stacked MoE decode tokens/s (%d layers)" % L, "value": steps * B / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (per-layer seeded BF16 weights; h0 ~ N(0,1))",
        "config": dict(config_of(w, args), k=k, budget=round(k / w.inter, 4), rank=rank, global_batch=B,
                       batch_per_gpu=B, replicas=1, layers=L, path=plan,
                       l2="inputs larger than L2: %.1f GB of packed weights" %
                          (sum(x.nbytes() for x in layers) / 1e9)),
        "us_per_layer": ms_per_step * 1e3 / L, "bytes_per_step": byts,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "traffic": None},
        # per step: L blocks and L + 1 residual/RMSNorm launches
        "gpu_launches": steps * (L * block_launches(plan["path"], dense, rank) + L + 1),
        "clocks": clk.summary(), "setup_s": setup_s,
    }
    print(json.dumps(line), flush=True)
    del graph


def run_threshold(args, w, world, rank, local):
    """The calibrated-threshold comparator on the same scores: tau is calibrated on
    held-out tokens for the budget k/I, then the decode steps read whatever passes."""
    import torch
    import token_top_expert_b200 as msb
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B = args.batch
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, args.rank, 1)
    layer = msb.PackedLayer.from_host(dims, msb.pack(lw.gate, lw.up, lw.down, lw.router, dims),
                                      lw.lr_a, lw.lr_b, device=dev)
    del lw
    ws = msb.Workspace(dims, max(B, 8), dev)
    # calibration: 256 held-out tokens, GPU scores of their routed experts
    pooled = []
    for i in range(32):
        xc = torch.from_numpy(synth.calibration_activations(w, i, 8).view(np.int16)).to(dev).view(torch.bfloat16)
        tr = msb.Trace(dims, 8, args.k, scores=True)
        msb.moe_sparse_block(xc, layer, args.k, workspace=ws, trace=tr, general=True)
        pooled.append(tr.scores[:, :, :w.inter].float().cpu().numpy().ravel())
    tau = msb.calibrate_threshold(np.concatenate(pooled), args.k / w.inter)
    nseq = 64
    xs = torch.from_numpy(np.stack([synth.activations(w, s, batch=B) for s in range(nseq)]).view(np.int16)).to(dev).view(torch.bfloat16)
    out = torch.empty_like(xs[0])
    # timed steps rotate over weight replicas, as the top-k bench does (inputs beyond L2)
    layers = [layer] + [layer.clone() for _ in range(args.replicas - 1)]
    counts = []
    byts = []
    tr = msb.Trace(dims, B, args.k, threshold=True)
    for s in range(nseq):
        msb.moe_sparse_block_threshold(xs[s], layer, tau, out=out, workspace=ws, trace=tr)
        torch.cuda.synchronize()
        counts.append(tr.sel_count.cpu().numpy().ravel().copy())
        byts.append(algorithmic_bytes(w, args.k, args.rank, tr.union_count.cpu().tolist(), False))
    counts = np.concatenate(counts) / w.inter
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            msb.moe_sparse_block_threshold(xs[s % nseq], layers[s % len(layers)], tau, out=out, workspace=ws,
                                           stream=stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for s in range(nseq):
            msb.moe_sparse_block_threshold(xs[s], layers[s % len(layers)], tau, out=out, workspace=ws,
                                           stream=stream)
    reps = max(1, args.steps // nseq)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / (reps * nseq)
    line = {"metric": "threshold comparator: read fraction per (token, expert) and tokens/s",
            "tau": tau, "budget": args.k / w.inter,
            "read_fraction": {"mean": float(counts.mean()), "std": float(counts.std()),
                              "min": float(counts.min()), "max": float(counts.max())},
            "value": B / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "batch": B,
            "bytes_per_step": float(np.mean(byts)), "config": config_of(w, args),
            "data": "synthetic; tau from 256 held-out tokens (weights and routing as the bench)",
            "l2": "inputs larger than L2: %d weight replicas rotated per step" % len(layers)}
    print(json.dumps(line), flush=True)
    del graph


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (one process each, under torchrun)")
    ap.add_argument("--steps", type=int, default=100000, help="timed decode steps")
    ap.add_argument("--warmup", type=int, default=20, help="untimed warm-up steps")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"],
                    help="ours: the CUDA library; reference: the FP64 CPU oracle on a bounded sample")
    ap.add_argument("--workload", default=synth.QWEN30B_BLOCK.name, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--k", type=int, default=None, help="channels kept per (token, expert)")
    ap.add_argument("--budget", type=float, default=None,
                    help="read budget as a fraction of I (k = round(budget * I)); --k wins")
    ap.add_argument("--batch", type=int, default=None, help="tokens per step")
    ap.add_argument("--rank", type=int, default=None, help="compensation rank r (0: none)")
    ap.add_argument("--replicas", type=int, default=8,
                    help="weight copies rotated per step so that every step reads HBM")
    ap.add_argument("--general", action="store_true", help="force the multi-kernel path")
    ap.add_argument("--single", action="store_true",
                    help="ask for the single-launch kernel (batches up to 16 tokens), even past "
                         "the measured crossover where the multi-kernel path is the default")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU-oracle timing")
    ap.add_argument("--e2e-steps", type=int, default=2000,
                    help="steps of the end-to-end measurement (host copies in the timed region)")
    ap.add_argument("--top-e", type=int, default=None,
                    help="route each token to this many experts (at most the trained count)")
    ap.add_argument("--stack-grid", action="store_true",
                    help="stacked workload: run k in {13%%, 18%%, 100%%} x batch in {1, 32} on one set of layers")
    ap.add_argument("--threshold", action="store_true",
                    help="measure the calibrated-threshold comparator instead of top-k")
    ap.add_argument("--q4", action="store_true",
                    help="4-bit channel records (moe_sparse_block_q4; batches of at most 16 tokens)")
    ap.add_argument("--phase-marks", action="store_true",
                    help="per-phase timeline of the single-launch kernel (instrumented build)")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.k is None and args.budget is not None:
        if not 0.0 < args.budget <= 1.0:
            ap.error("--budget must lie in (0, 1]")
        args.k = max(1, synth.budget_k(args.budget, w.inter))
    args.k = w.k if args.k is None else args.k
    args.batch = w.batch if args.batch is None else args.batch
    args.rank = w.rank if args.rank is None else args.rank
    if args.k == w.inter and args.rank == w.rank and "--rank" not in sys.argv:
        args.rank = 0  # the dense reference path has no compensation term
    world, rank, local = dist_setup()
    args.gpus = world if world > 1 else args.gpus

    if args.impl == "reference":
        run_reference(args, w, world, rank)
        return
    if args.phase_marks:
        os.environ["MSB_VARIANT"] = "instr"
        from token_top_expert_b200 import build as _bm
        _bm.build(variant="instr")
        run_phase_marks(args, w, local)
        return
    if w.layers > 1 or args.threshold:
        from token_top_expert_b200 import build as _bld
        _bld.build()
        if w.layers > 1:
            run_stack(args, w, world, rank, local)
        else:
            run_threshold(args, w, world, rank, local)
        return

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import token_top_expert_b200 as msb
    from token_top_expert_b200 import build as _b
    _b.build()
    msb.load_library()
    dev = torch.device("cuda", local)

    # ---- weights: generate, pack (host C++ packer), upload, replicate
    lw = synth.layer_weights(w)
    dims = msb.Dims(w.d, w.inter, w.experts, w.top_e, args.rank, 1)
    pk = (msb.pack_q4 if args.q4 else msb.pack)(lw.gate, lw.up, lw.down, lw.router, dims)
    base = msb.PackedLayer.from_host(dims, pk, lw.lr_a, lw.lr_b, device=dev)
    del lw, pk
    layers = [base] + [base.clone() for _ in range(args.replicas - 1)]
    B = args.batch
    nseq = min(w.steps, 1000)
    xs_host = [synth.activations(w, s, batch=B) for s in range(nseq)]
    xs = torch.from_numpy(np.stack(xs_host).view(np.int16)).to(dev).view(torch.bfloat16)
    outs = torch.empty_like(xs)
    ws = msb.Workspace(dims, B, dev)
    stream = torch.cuda.Stream(dev)
    general, single = args.general, args.single

    def step(i, s):
        msb.moe_sparse_block(xs[i % nseq], layers[i % args.replicas], args.k, out=outs[i % nseq],
                             workspace=ws, general=general, stream=s, top_e=args.top_e,
                             single=single)

    # ---- union sizes of every step of the sequence (one traced pass) -> algorithmic bytes
    dense = args.k == w.inter
    Kr = args.top_e or w.top_e
    # (4-bit records run on the single launch, which leaves a batch's union count to the
    # host: it is formed here from the traced selections)
    host_union = args.q4 and B > 1
    tr = msb.Trace(msb.Dims(w.d, w.inter, w.experts, Kr, args.rank, 1), B, args.k, union=not host_union)
    bytes_per_step = []
    with torch.cuda.stream(stream):
        for i in range(nseq):
            msb.moe_sparse_block(xs[i], layers[i % args.replicas], args.k, out=outs[i],
                                 workspace=ws, trace=tr, general=general, stream=stream,
                                 top_e=args.top_e)
            if i < 64 or not (B == 1 and not dense):
                stream.synchronize()
                if host_union:
                    ids, sel = tr.expert_ids.cpu().numpy(), tr.sel.cpu().numpy()
                    sets = {}
                    for t in range(B):
                        for r in range(Kr):
                            sets.setdefault(int(ids[t][r]), set()).update(sel[t][r].tolist())
                    union = [len(v) for v in sets.values()]
                else:
                    union = tr.union_count.cpu().tolist()
                bytes_per_step.append(algorithmic_bytes(w, args.k, args.rank, union, dense, args.q4))
    stream.synchronize()
    ws.check(stream)
    step_bytes = float(np.mean(bytes_per_step))
    router_bytes = 2 * w.d * w.experts

    # ---- warmup (untimed), then capture the decode sequence as one CUDA graph
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    G = min(nseq, args.steps)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            step(i, stream)
    tail = None
    if args.steps % G:
        tail = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tail, stream=stream):
            for i in range(args.steps % G):
                step(i, stream)
    graph.replay()
    stream.synchronize()

    # ---- timed region: exactly K steps
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]
                    if os.environ.get("CUDA_VISIBLE_DEVICES") else local)
    with ClockSampler(gpu_index) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps // G):
                graph.replay()
            if tail is not None:
                tail.replay()
            e1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    ms, value = replica_throughput(e0.elapsed_time(e1), args.steps * B, dist, dev)
    if dist is not None:
        dist.barrier()
    ms_per_step = ms / args.steps
    ws.check(stream)

    # ---- e2e: the C-ABI call on host buffers, per step: pinned host x -> device, the
    # block, device -> pinned host out (moe_sparse_block_host through HostCall; with
    # --top-e, the device call between two torch copies)
    xh = torch.from_numpy(np.stack(xs_host).view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    ne = min(args.e2e_steps, args.steps)
    if args.top_e is None and not args.q4:
        # the host produces each step's x before the call (nothing on the stream writes
        # it), so the calls declare it ready: the kernel fetches x across the host link
        # while the previous launch still runs
        calls = [msb.HostCall(lay, args.k, B, stream=stream, general=general, x_ready=True, single=single)
                 for lay in layers]
        xp = [xh[i].data_ptr() for i in range(nseq)]
        op = [oh[i].data_ptr() for i in range(nseq)]

        def e2e_step(i):
            calls[i % args.replicas](xp[i % nseq], op[i % nseq])
    else:
        xd = torch.empty((B, w.d), dtype=torch.bfloat16, device=dev)
        od = torch.empty_like(xd)

        def e2e_step(i):
            xd.copy_(xh[i % nseq], non_blocking=True)
            msb.moe_sparse_block(xd, layers[i % args.replicas], args.k, out=od, workspace=ws,
                                 general=general, stream=stream, top_e=args.top_e, single=single)
            oh[i % nseq].copy_(od, non_blocking=True)
    with torch.cuda.stream(stream):
        for i in range(min(50, ne)):
            e2e_step(i)
        stream.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(ne):
            e2e_step(i)
        a1.record(stream)
        stream.synchronize()
    e2e_ms, e2e_value = replica_throughput(a0.elapsed_time(a1), ne * B, dist, dev)
    # the host results of the last steps match the device results of the same steps (up to
    # the order of the FP32 reduction-adds across experts)
    for i in range(max(0, ne - 8), ne):
        a_, b_ = oh[i % nseq].float(), outs[i % nseq].float().cpu()
        if float((a_ - b_).norm()) > 1e-2 * float(b_.norm()):
            raise SystemExit("e2e output of step %d differs from the device-timed run" % i)

    peak, peak_kind = peaks()
    achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
    plan = msb.path_info(msb.Dims(w.d, w.inter, w.experts, args.top_e or w.top_e, args.rank, 1), B,
                         args.k, general=general, single=bool(args.q4) or single)  # 4-bit: single only
    kernel = "fused_block_kernel" if plan["path"] == "single_launch" else "multi_kernel_step"
    traffic = recorded_traffic(kernel, w.name + ("_dense" if dense else "") + ("_q4" if args.q4 else ""))
    launches_per_step = block_launches(plan["path"], dense, args.rank)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world if world > 1 else 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) BF16 weights, 5% rows x4; x ~ N(0,1))",
        "config": dict(config_of(w, args), path=plan),
        "us_per_block": ms_per_step * 1e3,
        "bytes_per_step": step_bytes, "router_bytes_per_step": router_bytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                     "kernel": kernel,
                     "note": "achieved = algorithmic bytes per step / device time per step "
                             "(CUDA events over the timed graph replays, launch gaps included)"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": B * w.d * 2,
                "d2h_bytes_per_step": B * w.d * 2, "steps": ne},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        v, ntok, dt, threads = oracle_sample(w, args.k, args.rank, xs_host, budget_s=6.0,
                                             top_e=args.top_e, q4=args.q4)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": "%d token-blocks: passes over the first tokens of the "
                                          "same decode sequence (FP64 numpy oracle, weights "
                                          "cached by an untimed pass), %.1f s" % (ntok, dt)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, tail
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
