"""CPU tests of bench.py's host logic: the multi-rank (replica) helpers over
gloo with world size 2, the per-rank input seeds, and the reference arm's
output contract."""
import dataclasses
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ring_context_parallelism_ra_b200.workloads import make_workload_inputs, workload  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world)
        out_q.put((rank, got))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


def test_replica_seeds_give_different_inputs():
    wl = workload("noncausal_fp32_512")
    q0, _, _ = make_workload_inputs(wl)
    q1, _, _ = make_workload_inputs(dataclasses.replace(wl, seed=wl.seed + 1000))
    q0b, _, _ = make_workload_inputs(wl)
    assert torch.equal(q0, q0b)
    assert not torch.equal(q0, q1)


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line():
    env = dict(os.environ, RA_ORACLE_BUDGET_S="0.6")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
    # the headline workload is the largest causal prefill (the MLA-shaped 256K)
    wl = workload("causal_mla_256k")
    assert line["config"] == bench.config_of(wl, 1)
    # a step is a bounded sample: its measured wall time, not the extrapolation
    assert line["ms_per_step"] < 10_000 < line["ms_per_step_full_workload_extrapolated"]


def test_flop_and_byte_counts_match_oracle_formulas():
    from oracle.costs import backward_flops as oracle_bwd_flops
    from oracle.costs import kv_cache_bytes, prefill_flops as oracle_flops
    from ring_context_parallelism_ra_b200.workloads import (backward_flops, decode_kv_bytes,
                                                           prefill_flops)
    for key in ("noncausal_fp32_512", "causal_mha_8k", "causal_gqa_128k", "causal_mla_256k"):
        wl = workload(key)
        assert prefill_flops(wl) == oracle_flops(wl.B, wl.n, wl.d_qk, wl.d_v, wl.Hq, wl.causal)
        assert backward_flops(wl) == oracle_bwd_flops(wl.B, wl.n, wl.d_qk, wl.d_v, wl.Hq,
                                                      wl.causal)
    wl = workload("decode_1m")
    assert decode_kv_bytes(wl) == wl.B * kv_cache_bytes(1, wl.Hkv, wl.d_qk, wl.n, 2)
    assert decode_kv_bytes(wl) == 17179869184


def test_kernel_source_hash_follows_code_not_comments():
    a = "int f(int x) {  // doubles\n  return 2 * x; /* fast */ }\n"
    b = "/* header */ int f(int x) {\n    return 2 * x;\n}  // end\n"
    c = "int f(int x) { return 3 * x; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_committed_traffic_matches_current_kernel_sources():
    # profiles/traffic.json holds DRAM bytes captured on the kernels' current
    # code; the bench reports them only while the code is unchanged
    assert bench.load_traffic("ring_forward:causal_mha_b1_h8_n8192_d128_P4", bench.TC_FILES)
    assert bench.load_traffic("ring_backward:causal_mha_b1_h8_n8192_d128_P4", bench.BWD_FILES)


def test_recap_carries_every_leg_in_a_short_tail():
    # a line shaped like the GPU arm's: the recap repeats each leg's value and
    # fraction, and with the decode leg after it the last 1500 characters hold
    # recap, decode and the decode short-cache latencies
    def entry(name, value, frac):
        return {"workload": name, "value": value, "roofline": {"frac": frac, "pad": "x" * 400}}
    line = {"value": 1100.0, "roofline": {"frac": 0.67}, "config": {"workload": "w5"},
            "e2e": {"value": 1050.0},
            "workloads": [entry("w3", 1000.0, 0.61), entry("w2", 900.0, 0.55)],
            "backward": [entry("w5", 760.0, 0.46), entry("w3", 850.0, 0.52)],
            "merge": [{"value": 2500.0}, {"value": 6100.0}],
            "striped": {"ring_speedup_striped_over_contiguous": 1.78},
            "cpu_baseline": {"value": 0.01, "sample": "y" * 300},
            "decode_short_cache": {"tokens": 32768, "pad": "z" * 150},
            "decode": {"value": 6900.0, "pad": "d" * 400}}
    r = bench.recap(line)
    assert r["prefill"] == {"w5": [1100.0, 0.67], "w3": [1000.0, 0.61], "w2": [900.0, 0.55]}
    assert r["backward"] == {"w5": [760.0, 0.46], "w3": [850.0, 0.52]}
    assert r["e2e_tflops"] == 1050.0 and r["merge_gbs"] == [2500.0, 6100.0]
    line["recap"] = r
    for key in ("decode_short_cache", "decode"):
        line[key] = line.pop(key)
    tail = json.dumps(line)[-1500:]
    assert '"recap"' in tail and '"decode"' in tail
