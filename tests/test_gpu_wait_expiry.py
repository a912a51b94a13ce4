"""A bounded device wait that runs out is reported, and the library recovers.

Every wait of the kernels on an mbarrier is bounded; when one runs out the kernel sets
the sticky error word, waits (bounded) for its own copies in flight, keeps every
exchange and barrier step, and finishes.  The instrumented build can withhold one bulk
copy on purpose (it is simply never issued: no bad address, no fault), so the wait for
it runs out after a 50 us limit.  tests/instrumented_check.py does this in a process of
its own, on both paths; here we check that msb_check reports MSB_ETIMEOUT for that call
and MSB_OK for the next one on the same workspace, whose output matches the oracle.
"""
import json
import os
import subprocess
import sys

import pytest

from parity import OUT_RTOL

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_wait_expiry_is_flagged_then_recovers():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    p = subprocess.run([sys.executable, os.path.join(HERE, "instrumented_check.py")],
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stdout + p.stderr
    res = json.loads(p.stdout.strip().splitlines()[-1])
    assert res["single_launch"]["path"] == "single_launch"
    assert res["general"]["path"] == "multi_kernel"
    for name, r in res.items():
        assert r["sabotaged_status"] == -4, (name, r)   # MSB_ETIMEOUT
        assert r["next_status"] == 0, (name, r)
        assert r["next_max_rel_l2"] <= OUT_RTOL, (name, r)
    print(res)
