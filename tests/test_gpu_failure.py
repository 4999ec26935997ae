"""Failure detection on the GPU without a fault: the grouped GEMM's bounded waits.

A child process runs with two test hooks of the library set in its environment: a short
wait limit (20 ms) and the second pipeline stage, which CTA 0's producer skips (no load, no arrival).
The MMA warp's wait for that stage runs out; the kernel must record MOE_ERR_TIMEOUT in the
workspace status word, drain its copies and MMAs, free TMEM and return, leaving the context
usable.  Nothing traps, faults or hangs.
"""

import json
import os
import subprocess
import sys

import pytest

from mixture_experts_layer_offsets_b200 import capi

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("dtype", ["bf16", "mxfp8"])
@pytest.mark.timeout(120)
def test_dropped_stage_times_out_cleanly(dtype):
    env = dict(os.environ, MOE_B200_WAIT_NS="20000000", MOE_B200_TEST_DROP_STAGE="2")
    out = subprocess.run([sys.executable, os.path.join(HERE, "failure_child.py"), dtype], env=env,
                         capture_output=True, text=True, timeout=100)
    assert out.returncode == 0, out.stderr[-2000:]
    res = json.loads(out.stdout.strip().splitlines()[-1])
    assert res["status"] == capi.MOE_ERR_TIMEOUT
    assert res["usable_after"]
    assert res["elapsed_s"] < 10.0
