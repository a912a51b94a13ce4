"""ctypes loader of libmsb.so (the C ABI declared in include/msb.h and include/msb_q4.h).

Loading fails loudly: there is no fallback implementation of any step.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MSB_VARIANT=instr selects the instrumented build (phase marks, wait-expiry injection)
VARIANT = os.environ.get("MSB_VARIANT") or None
LIB_PATH = os.path.join(_HERE, "libmsb_instr.so" if VARIANT == "instr" else "libmsb.so")

MSB_OK = 0
MSB_EINVAL = -1
MSB_EUNSUPPORTED = -2
MSB_ECUDA = -3
MSB_ETIMEOUT = -4
MSB_ENONFINITE = -5
MSB_EINTERNAL = -6
MSB_FLAG_GENERAL = 1
MSB_FLAG_X_READY = 2
MSB_FLAG_SINGLE = 4

MSB_MAX_D = 8192
MSB_MAX_INTER = 4096
MSB_MAX_EXPERTS = 512
MSB_MAX_TOP_E = 16
MSB_MAX_RANK = 128
MSB_MAX_BATCH = 256

# every function include/msb.h and include/msb_q4.h declare
SYMBOLS = (
    "msb_sketch_words", "msb_alpha_count", "msb_pack", "msb_ternary_rows", "msb_workspace_size",
    "msb_workspace_init", "msb_check", "msb_strerror", "moe_sparse_block",
    "moe_sparse_block_threshold", "msb_residual_rmsnorm", "msb_path_info",
    "moe_sparse_block_noalloc", "msb_noalloc_check", "moe_sparse_block_top_e",
    "moe_sparse_block_host",
    "msb_q4_record_bytes", "msb_pack_q4", "moe_sparse_block_q4",
)
MSB_Q4_GROUP = 64


class MsbDims(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("inter", ctypes.c_int32), ("experts", ctypes.c_int32),
                ("top_e", ctypes.c_int32), ("rank", ctypes.c_int32), ("renorm", ctypes.c_int32)]


class MsbTrace(ctypes.Structure):
    _fields_ = [("expert_ids", ctypes.c_void_p), ("expert_w", ctypes.c_void_p),
                ("sel", ctypes.c_void_p), ("sel_count", ctypes.c_void_p),
                ("union_count", ctypes.c_void_p), ("scores", ctypes.c_void_p)]


class MsbError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = _lib.msb_strerror(status).decode() if _lib is not None else str(status)
        super().__init__("%s failed: %s (status %d)" % (what or "msb call", msg, status))


_lib = None


def load() -> ctypes.CDLL:
    """Load libmsb.so once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("%s is not built; run `python -m token_top_expert_b200.build%s`"
                          % (LIB_PATH, " --instrumented" if VARIANT == "instr" else ""))
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, U32, SZ, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t, ctypes.c_float
    dims_p = ctypes.POINTER(MsbDims)
    trace_p = ctypes.POINTER(MsbTrace)
    sig = {
        "msb_sketch_words": (SZ, [dims_p]),
        "msb_alpha_count": (SZ, [dims_p]),
        "msb_pack": (I32, [P, P, P, P, dims_p, P, P, P, P, I32]),
        "msb_ternary_rows": (I32, [P, I32, I32, P, P]),
        "msb_q4_record_bytes": (SZ, [dims_p]),
        "msb_pack_q4": (I32, [P, P, P, P, dims_p, P, P, P, P, I32]),
        "msb_workspace_size": (SZ, [dims_p, I32]),
        "msb_workspace_init": (I32, [P, SZ, P]),
        "msb_check": (I32, [P, P]),
        "msb_strerror": (ctypes.c_char_p, [I32]),
        "moe_sparse_block": (I32, [P, I32, P, P, P, P, I32, P, P, P, dims_p, P, SZ, trace_p, U32, P]),
        "moe_sparse_block_q4": (I32, [P, I32, P, P, P, P, I32, P, P, P, dims_p, P, SZ, trace_p, U32, P]),
        "moe_sparse_block_threshold": (I32, [P, I32, P, P, P, P, F32, P, P, P, dims_p, P, SZ,
                                             trace_p, P]),
        "msb_residual_rmsnorm": (I32, [P, P, P, I32, I32, F32, P]),
        "msb_path_info": (I32, [dims_p, I32, I32, U32, P]),
        "moe_sparse_block_noalloc": (I32, [P, P, P, P, P, I32, P, P, P, dims_p, trace_p, P]),
        "msb_noalloc_check": (I32, [P]),
        "moe_sparse_block_top_e": (I32, [P, I32, P, P, P, P, I32, I32, P, P, P, dims_p, P, SZ,
                                         trace_p, U32, P]),
        "moe_sparse_block_host": (I32, [P, P, I32, P, P, P, P, I32, P, P, P, P, dims_p, P, SZ,
                                        U32, P]),
    }
    if VARIANT == "instr":
        sig["msb_debug_set_marks"] = (I32, [P])
        sig["msb_debug_inject"] = (I32, [U32, ctypes.c_uint64])
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
