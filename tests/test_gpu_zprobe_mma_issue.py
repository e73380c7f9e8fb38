"""GPU check of a property of the hardware that the kernels' MMA-issue design
relies on: one lane can keep the tensor pipe busy with M = 128, K = 16
tcgen05.mma instructions -- 64 cycles each at N = 128, 128 at N = 256 --
issuing batches whose B operand moves between shared-memory slots, as the
kernels do with their K/V ring.  The probe (tests/probes/mma_issue_probe.cu,
built here with nvcc against the library's PTX wrappers) also reports the
converged-warp form (one elected lane per instruction) and descriptors formed
ahead of the batch, for the record.  A second probe
(tests/probes/mma_operand_probe.cu) times the operand forms the kernels use:
every K-major / MN-major / tensor-memory combination at N = 128 runs at the
same 64 cycles, while N = 64 takes more than half of an N = 128 instruction
(so splitting a product into N = 64 halves costs tensor time).  This file
runs after the parity tests.
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


def _run_probe(name):
    from ring_context_parallelism_ra_b200 import build as B
    src = os.path.join(ROOT, "tests", "probes", name + ".cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, name)
        subprocess.run([B.nvcc(), *B.ARCH, "-O3", "-std=c++17", "-I",
                        os.path.join(ROOT, "ring_context_parallelism_ra_b200", "csrc"),
                        "-o", exe, src], check=True, capture_output=True, timeout=300)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    res = json.loads(r.stdout.strip().splitlines()[-1])
    print(res)
    return res


def test_one_lane_issues_tcgen05_mma_at_the_tensor_pipe_rate():
    res = _run_probe("mma_issue_probe")
    assert res["timeouts"] == 0
    assert res["lane0_inline"] <= 1.25 * 64, res
    assert res["lane0_inline_n256"] <= 1.25 * 128, res


def test_operand_forms_run_at_one_rate_and_n64_is_not_half_an_n128():
    res = _run_probe("mma_operand_probe")
    assert res["timeouts"] == 0
    for form in ("ss_kk", "ss_k_mn", "ss_mn_mn", "ts_b_mn", "ts_b_k"):
        assert res[form] <= 1.25 * 64, res
    # an N = 64 instruction takes well over half the time of an N = 128 one
    assert res["ss_kk_n64"] > 0.7 * res["ss_kk"], res
