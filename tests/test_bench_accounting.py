"""The bench's algorithmic byte count (the roofline's numerator) against the oracle's
definition of the bytes one step must read, and the stated per-step totals."""
import importlib.util
import os

import numpy as np

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bytes_match_the_oracle_definition():
    bench = _bench()
    w = synth.QWEN30B_BLOCK
    # batch 1, k = 138: 8 used experts of 128 (the trace reports 0 for the others)
    unions = [0] * 120 + [138] * 8
    assert bench.algorithmic_bytes(w, 138, 32, unions, False) == 18_833_408
    assert oracle.read_bytes([138] * 8, w.d, w.inter, 32) == 18_833_408
    # dense block (k = I, r = 0): channel records only
    assert bench.algorithmic_bytes(w, 768, 0, [0] * 120 + [768] * 8, True) == 75_497_472
    assert oracle.read_bytes([768] * 8, w.d, w.inter, 0, dense=True) == 75_497_472
    # batch: unions of varying size, any rank
    rng = np.random.default_rng(0)
    for r in (0, 16, 64):
        u = [int(v) for v in rng.integers(1, w.inter, 40)]
        assert bench.algorithmic_bytes(w, 100, r, u + [0] * 88, False) == \
            oracle.read_bytes(u, w.d, w.inter, r)
    # k = I with compensation: records plus A_e, B_e, no sketch
    assert bench.algorithmic_bytes(w, 768, 32, [768] * 8, True) == 8 * (6 * 2048 * 768 + 4 * 2048 * 32)


def test_large_block_and_budget_totals():
    bench = _bench()
    w = synth.LARGE_BLOCK
    assert bench.algorithmic_bytes(w, 276, 64, [276] * 8, False) == 75_284_480


def test_launch_counts_follow_the_launch_sequence():
    """One launch on the single-launch path; on the multi-kernel path router, score
    (skipped for a dense block without compensation), select (skipped when dense),
    union, gather, finalize."""
    bench = _bench()
    assert bench.block_launches("single_launch", False, 32) == 1
    assert bench.block_launches("multi_kernel", False, 32) == 6
    assert bench.block_launches("multi_kernel", False, 0) == 6
    assert bench.block_launches("multi_kernel", True, 0) == 4
    assert bench.block_launches("multi_kernel", True, 32) == 5
