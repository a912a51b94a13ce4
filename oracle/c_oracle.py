"""ctypes wrapper of the plain C99 restatement in ``oracle/c/msb_oracle.c`` (TEST
INFRASTRUCTURE, like the rest of ``oracle``): a second, independently written oracle
that the tests hold against the numpy one.

The shared library is compiled on first use with gcc (-O2, no fast-math, no FP
contraction) into ``oracle/c/libmsb_oracle.so``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "c")
SRC = os.path.join(_DIR, "msb_oracle.c")
LIB = os.path.join(_DIR, "libmsb_oracle.so")
CMD = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
       "-Wall", "-Wextra", "-Werror", SRC, "-o", LIB, "-lm"]

_lib = None


def build() -> str:
    """Compile the C oracle if its library is missing or older than its source."""
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(CMD, check=True, capture_output=True, text=True)
    return LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.msb_oracle_block.restype = I
        lib.msb_oracle_block.argtypes = [P, I, P, P, P, P, P, P, I, I, I, I, I, I, I, I, D,
                                         P, P, P, P, P, P]
        _lib = lib
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16
    return a


def moe_block(x_bits, gate, up, down, router, top_e, k=None, lr_a=None, lr_b=None, renorm=True,
              mode="topk", tau=0.0):
    """One block step by the C oracle.  All arrays are BF16 bits in model layout:
    x [B][d], gate/up [E][I][d], down [E][d][I], router [d][E], lr_a [E][d][r],
    lr_b [E][r][d].  mode: "topk", "threshold" or "dense".  Returns a dict like
    ``oracle.moe_block``: y [B][d], ids [B][K], w [B][K], sel {(t, e): channels},
    scores {(t, e): s} (not in dense mode)."""
    x_bits, gate, up, down, router = map(_u16, (x_bits, gate, up, down, router))
    B, d = x_bits.shape
    E, I, _ = gate.shape
    K = top_e
    r = 0 if lr_a is None else lr_a.shape[2]
    if r:
        lr_a, lr_b = _u16(lr_a), _u16(lr_b)
    m = {"topk": 0, "threshold": 1, "dense": 2}[mode]
    y = np.zeros((B, d))
    ids = np.zeros((B, K), np.int32)
    w = np.zeros((B, K))
    sel = np.zeros((B, K, I), np.int32)
    nsel = np.zeros((B, K), np.int32)
    scores = np.zeros((B, K, I))
    ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
    rc = _load().msb_oracle_block(ptr(x_bits), B, ptr(router), ptr(gate), ptr(up), ptr(down),
                                  ptr(lr_a), ptr(lr_b), d, I, E, K, r, int(renorm), m,
                                  0 if k is None else int(k), float(tau), ptr(y), ptr(ids), ptr(w),
                                  ptr(sel), ptr(nsel), ptr(scores))
    if rc != 0:
        raise ValueError("msb_oracle_block rejected its arguments")
    out = {"y": y, "ids": ids, "w": w, "sel": {}, "scores": {}}
    for t in range(B):
        for q in range(K):
            e = int(ids[t, q])
            out["sel"][(t, e)] = sel[t, q, :nsel[t, q]].astype(np.int64)
            if mode != "dense":
                out["scores"][(t, e)] = scores[t, q]
    return out
