"""Build libmsb.so in-tree with nvcc for sm_100a (B200).

    python -m token_top_expert_b200.build

Every .cu / .cpp file under csrc/ is compiled to an object in _build/ (in
parallel) and linked into token_top_expert_b200/libmsb.so.  The CUDA runtime is
linked statically, so the library loads on a machine without a GPU (the host
packer and the argument checks work there).

    python -m token_top_expert_b200.build --instrumented

builds the instrumented variant libmsb_instr.so (objects in _build_instr/): the same
sources with MSB_INSTRUMENTED defined.  Its single-launch kernel records a
%globaltimer mark per phase and CTA (read by `bench.py --phase-marks`), and a test can
make one bounded wait run out on purpose (`msb_debug_inject`; tests/instrumented_check.py).
The product library is built without either.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmsb.so")
VARIANTS = {None: (BUILD, LIB, []),
            "instr": (os.path.join(PKG, "_build_instr"), os.path.join(PKG, "libmsb_instr.so"),
                      ["-DMSB_INSTRUMENTED"])}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, ptxas_verbose: bool = False, variant: str | None = None) -> str:
    """Compile and link; returns the library path.  Raises on any compiler error."""
    BUILD, LIB, defs = VARIANTS[variant]
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    cc = nvcc()
    jobs = []
    objs = []
    for src in _sources():
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if _newer(obj, [path] + headers):
            continue
        cmd = [cc] + ARCH + COMMON + defs + ["-c", path, "-o", obj]
        if ptxas_verbose and src.endswith(".cu"):
            cmd += ["-Xptxas", "-v"]
        jobs.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        p = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, p

    with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
        for cmd, p in ex.map(run, jobs):
            if verbose or ptxas_verbose:
                sys.stdout.write(p.stdout + p.stderr)
            if p.returncode != 0:
                raise RuntimeError("compile failed: %s\n%s%s" % (" ".join(cmd), p.stdout, p.stderr))
    if not _newer(LIB, objs):
        cmd = [cc] + ARCH + ["-shared", "-o", LIB] + objs + ["-lpthread"]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError("link failed: %s\n%s%s" % (" ".join(cmd), p.stdout, p.stderr))
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, ptxas_verbose="--ptxas" in sys.argv,
                variant="instr" if "--instrumented" in sys.argv else None))
