"""GPU check of a property of the hardware that the kernels' MMA-issue design
relies on: one lane can keep the tensor pipe busy with M = 128, K = 16
tcgen05.mma instructions -- 64 cycles each at N = 128, 128 at N = 256 --
issuing batches whose B operand moves between shared-memory slots, as the
kernels do with their K/V ring.  The probe (tests/probes/mma_issue_probe.cu,
built here with nvcc against the library's PTX wrappers) also reports the
converged-warp form (one elected lane per instruction) and descriptors formed
ahead of the batch, for the record.  This file runs after the parity tests.
"""
import json
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.gpu


def test_one_lane_issues_tcgen05_mma_at_the_tensor_pipe_rate():
    from ring_context_parallelism_ra_b200 import build as B
    src = os.path.join(ROOT, "tests", "probes", "mma_issue_probe.cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "mma_issue_probe")
        subprocess.run([B.nvcc(), *B.ARCH, "-O3", "-std=c++17", "-I",
                        os.path.join(ROOT, "ring_context_parallelism_ra_b200", "csrc"),
                        "-o", exe, src], check=True, capture_output=True, timeout=300)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    res = json.loads(r.stdout.strip().splitlines()[-1])
    print(res)
    assert res["timeouts"] == 0
    assert res["lane0_inline"] <= 1.25 * 64, res
    assert res["lane0_inline_n256"] <= 1.25 * 128, res
