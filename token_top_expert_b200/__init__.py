"""B200-native sparse-MoE block decode with calibration-free top-k channel selection.

The compute path is libmsb.so (hand-written sm_100a CUDA behind the C ABI in
include/msb.h); this package only marshals arguments to it.
"""
from ._lib import MsbError, load as load_library  # noqa: F401
from .block import (  # noqa: F401
    Dims,
    HostCall,
    PackedLayer,
    Trace,
    Workspace,
    calibrate_threshold,
    moe_sparse_block,
    moe_sparse_block_noalloc,
    moe_sparse_block_threshold,
    noalloc_check,
    pack,
    pack_q4,
    q4_record_bytes,
    path_info,
    residual_rmsnorm,
    sketch_words,
    workspace_size,
)
from . import checkpoint, lowrank, packfile  # noqa: F401,E402
