#!/usr/bin/env python3
"""Benchmark of the Ring Attention hot path on B200.

One step = one fused ring forward (all partitions, ring order, causal skip,
online-softmax fold, epilogue) over one batch of synthetic input of the
chosen workload.  The JSON line reports causal-adjusted TFLOP/s, the
roofline of the dominant kernel, the end-to-end number through the public
API from pinned host buffers, the oracle's CPU throughput on a bounded
sample, and the pass-Q decode leg (GB/s of KV cache read) that the metric
also names.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload causal_mla_256k|causal_gqa_128k|causal_mha_8k|noncausal_fp32_512]
    python bench.py --impl reference ...   # the fp64 CPU oracle, same line

N > 1 (torchrun): every rank runs an independent replica of the workload
(different seed), no collective on the data path; value = work of all ranks
divided by the slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ring_context_parallelism_ra_b200 import ra  # noqa: E402
from ring_context_parallelism_ra_b200.workloads import (decode_kv_bytes, make_workload_inputs,  # noqa: E402
                                                        prefill_flops, workload)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20   # > 126 MB L2
METRIC = "causal attn TFLOP/s & % BF16 peak (prefill ring); decode GB/s & % HBM peak"


# ---------------------------------------------------------------- helpers --

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text):
    """Source text without comments and with whitespace collapsed, so that a
    hash of it changes with the code and not with its commentary."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "ring_context_parallelism_ra_b200", "csrc", f),
                  encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel_key, files):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_sha") != kernel_source_sha(files):
        return None
    return e


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index, period_s=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nv = None
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvml unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world != n_gpus and world > 1:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE {world}", file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ cpu oracle --

def oracle_sample(wl, budget_s, seed=0):
    """Time the fp64 oracle on a bounded sample of query rows of the workload
    (drawn on the CPU with the workload recipe).  Returns (TFLOP/s, cores,
    description)."""
    from oracle.attention import attention as oracle_attention  # test infrastructure
    from ring_context_parallelism_ra_b200.workloads import make_qkv
    cores = len(os.sched_getaffinity(0))
    n = wl.n
    # one head-pair of the workload at full length (K, V of one KV head)
    q, k, v = make_qkv(1, 1, 1, n, n, wl.d_qk, wl.d_v, wl.torch_dtype, wl.seed + 77, wl.qk_mult)
    rng = np.random.default_rng(seed)
    done_rows, flops, t0 = 0, 0.0, time.perf_counter()
    chunk = max(8, min(512, 2 ** 22 // n))
    while time.perf_counter() - t0 < budget_s:
        rows = np.sort(rng.integers(0, n, chunk))
        oracle_attention(q, k, v, wl.scale, wl.causal, rows=rows)
        vis = (rows + 1) if wl.causal else np.full(len(rows), n)
        flops += float(2.0 * vis.sum() * (wl.d_qk + wl.d_v))
        done_rows += len(rows)
    dt = time.perf_counter() - t0
    desc = (f"{done_rows} random query rows of one head at n={n} (full key range each, "
            f"causal FLOPs counted per row), {dt:.1f} s")
    return flops / dt / 1e12, cores, desc, dt


# ------------------------------------------------------------- our arm ----

def run_ours(args, world, rank):
    dev = torch.device("cuda")
    wl = workload(args.workload)
    peaks, peaks_kind = load_peaks()
    flops = prefill_flops(wl)
    ra.lib()

    # each replica draws its own inputs (seed offset by rank)
    q, k, v = make_workload_inputs(dataclasses.replace(wl, seed=wl.seed + 1000 * rank), device=dev)
    out = torch.empty((wl.B, wl.Hq, wl.n, wl.d_v), device=dev, dtype=wl.torch_dtype)
    lse = torch.empty((wl.B, wl.Hq, wl.n), device=dev, dtype=torch.float32)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ra.ring_forward(q, k, v, wl.P, wl.causal, wl.scale, out, lse)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert ra.get_status() == ra.RA_OK

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = ra.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.zero_()                     # L2 flush between timed steps (not timed)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    launches = ra.launch_count() - launches0
    assert ra.get_status() == ra.RA_OK
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_local = statistics.mean(per_step)
    ms = max_over_ranks(ms_local, world)
    value = world * flops / (ms * 1e-3) / 1e12

    # roofline of the dominant (only) kernel of the step: one launch per step
    kernel_files = ["simt_attention.cu"] if wl.dtype == "f32" else TC_FILES
    achieved = flops / (ms_local * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tr = load_traffic(f"ring_forward:{wl.name}", kernel_files)
    roofline = {"bound": "tensor" if wl.dtype == "bf16" else "alu", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": tr["dram_bytes_per_launch"] if tr else None,
                "peak_kind": f"{peaks_kind} bf16 burst", "kernel": "ring_forward",
                "frac_of_sustained": round(achieved / peaks.get("bf16_tflops_sustained", 1400.0), 4)}
    if wl.dtype == "f32":  # the exact-fp32 path runs on the CUDA cores, not the tensor cores
        mhz = clk.summary().get("sm_max_mhz") or 1965
        num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
        peak = alu_peak_tflops(mhz, num_sms)
        roofline.update({"peak": round(peak, 2), "frac": round(achieved / peak, 4),
                         "peak_kind": f"fp32 FMA: {num_sms} SMs x 128 lanes x 2 FLOP x {mhz} MHz",
                         "frac_of_sustained": None})

    # end to end through the C ABI on host buffers: every step is one
    # ra_ring_forward_host call (Q, K, V copied in from pinned host memory,
    # the ring, O and LSE copied back), the copies of one chunk of heads
    # overlapping the kernels of its neighbours inside the call
    qh = q.cpu().pin_memory()
    kh = k.cpu().pin_memory()
    vh = v.cpu().pin_memory()
    del q, k, v, out, lse
    torch.cuda.empty_cache()
    out_h = torch.empty((wl.B, wl.Hq, wl.n, wl.d_v), dtype=wl.torch_dtype, pin_memory=True)
    lse_h = torch.empty((wl.B, wl.Hq, wl.n), dtype=torch.float32, pin_memory=True)
    ws = torch.empty(ra.ring_forward_host_workspace_bytes(qh, kh, vh), dtype=torch.uint8,
                     device=dev)

    def host_step():
        ra.ring_forward_host(qh, kh, vh, wl.P, wl.causal, wl.scale, out_h, lse_h, ws,
                             stream=stream, synchronize=False)

    for _ in range(3):
        host_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 20))
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        host_step()
    e1.record(stream)
    torch.cuda.synchronize()
    assert ra.get_status() == ra.RA_OK
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    e2e = {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
           "api": "ra_ring_forward_host (one C-ABI call per step: copies in, ring, copies out)"}
    del qh, kh, vh, out_h, lse_h, ws, flush
    torch.cuda.empty_cache()

    decode = None if args.skip_decode else run_decode_leg(args, world, rank, peaks, peaks_kind)
    striped = None if args.skip_striped else run_striped_leg(args, world, rank, workload("causal_gqa_128k"), peaks)
    merge = None if args.skip_merge else run_merge_leg(args, world, rank, peaks, peaks_kind)
    others = (None if args.skip_workloads
              else run_workloads_leg(args, world, rank, args.workload, peaks, peaks_kind))
    backward = None
    if not args.skip_backward:
        backward = [run_backward_leg(args, world, rank, workload(key), peaks, peaks_kind)
                    for key in BACKWARD_WORKLOADS]

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": config_of(wl, world),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if striped is not None:
        line["striped"] = striped
    if backward is not None:
        line["backward"] = backward
    if merge is not None:
        line["merge"] = merge
    if others is not None:
        line["workloads"] = others
    if decode is not None:
        # the pass-Q decode leg goes at the end of the line (main() keeps it
        # there), its short-cache latencies just before it
        line["decode_short_cache"] = decode.pop("short_cache")
        line["decode"] = decode
    return line


def recap(line):
    """Every leg's headline figure in a few hundred characters, placed near
    the end of the line (with the decode leg after it) so that a log that
    keeps only the line's tail still carries them: value and fraction of the
    measured peak per prefill and backward workload, end to end, merge."""
    def short(entry):
        return [entry["value"], entry["roofline"]["frac"]]
    r = {"prefill": {line["config"]["workload"]: [line["value"], line["roofline"]["frac"]]},
         "e2e_tflops": line["e2e"]["value"]}
    for w in line.get("workloads", []):
        r["prefill"][w["workload"]] = short(w)
    if "backward" in line:
        r["backward"] = {b["workload"]: short(b) for b in line["backward"]}
    if "merge" in line:
        r["merge_gbs"] = [m["value"] for m in line["merge"]]
    if "striped" in line:
        r["striped_ring_speedup"] = line["striped"].get("ring_speedup_striped_over_contiguous")
    r["format"] = "workload: [value, fraction of the measured peak]"
    return r


def config_of(wl, world):
    """The line's `config`; both arms print the same dict for a workload."""
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "seq_len": wl.n,
            "d_qk": wl.d_qk, "d_v": wl.d_v, "P": wl.P, "causal": wl.causal,
            "flops_per_step": prefill_flops(wl),
            "flop_convention": "2*B*Hq*n^2*(d_qk+d_v), x1/2 causal",
            "l2": "GPU arm: flushed between timed steps (256 MiB write, outside the step "
                  "events); CPU oracle arm: not applicable",
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def alu_peak_tflops(sm_mhz, num_sms):
    """fp32 FMA peak of the CUDA cores (not the tensor cores): 128 fp32 lanes
    per SM, 2 FLOP per FMA, at the given SM clock."""
    return num_sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def run_workloads_leg(args, world, rank, main_key, peaks, peaks_kind):
    """The fused ring forward on the other configured workloads (the fp32
    correctness shape, causal GQA 128K, causal MLA 256K), each timed like the
    main leg: warm-up, L2 flushed before every step, CUDA events on the
    launching stream, SM clocks sampled while timing."""
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    res = []
    for key in PREFILL_WORKLOADS:
        if key == main_key:
            continue
        wl = workload(key)
        flops = prefill_flops(wl)
        q, k, v = make_workload_inputs(dataclasses.replace(wl, seed=wl.seed + 1000 * rank), device=dev)
        out = torch.empty((wl.B, wl.Hq, wl.n, wl.d_v), device=dev, dtype=wl.torch_dtype)
        lse = torch.empty((wl.B, wl.Hq, wl.n), device=dev)
        steps = 10 if wl.n <= 8192 else 3
        for _ in range(3):
            flush.zero_()
            ra.ring_forward(q, k, v, wl.P, wl.causal, wl.scale, out, lse)
        torch.cuda.synchronize()
        events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
        barrier(world)
        with ClockSampler(torch.cuda.current_device()) as clk:
            for e0, e1 in events:
                flush.zero_()
                e0.record(stream)
                ra.ring_forward(q, k, v, wl.P, wl.causal, wl.scale, out, lse)
                e1.record(stream)
            torch.cuda.synchronize()
        assert ra.get_status() == ra.RA_OK
        ms_local = statistics.mean(e0.elapsed_time(e1) for e0, e1 in events)
        ms = max_over_ranks(ms_local, world)
        achieved = flops / (ms_local * 1e-3) / 1e12
        clocks = clk.summary()
        if wl.dtype == "bf16":
            peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
            sus = peaks.get("bf16_tflops_sustained")
            roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "frac_of_sustained": round(achieved / sus, 4) if sus else None,
                    "peak_kind": f"{peaks_kind} bf16 burst", "kernel": "tc_attention_kernel"}
        else:
            mhz = clocks.get("sm_max_mhz") or 1965
            peak = alu_peak_tflops(mhz, num_sms)
            roof = {"bound": "alu", "achieved": round(achieved, 3), "peak": round(peak, 2),
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_kind": f"fp32 FMA: {num_sms} SMs x 128 lanes x 2 FLOP x {mhz} MHz",
                    "kernel": "simt_attention_kernel",
                    "note": "correctness shape (512 tokens); its time is launch-dominated"}
        res.append({"workload": wl.name, "value": round(world * flops / (ms * 1e-3) / 1e12, 3),
                    "unit": "TFLOP/s", "ms_per_step": round(ms, 5), "steps": steps, "warmup": 3,
                    "dtype": "bf16" if wl.dtype == "bf16" else "f32", "roofline": roof,
                    "clocks": clocks})
        del q, k, v, out, lse
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return res


def run_merge_leg(args, world, rank, peaks, peaks_kind):
    """ra_lse_merge alone on the partials one query partition of a ring
    collects (P normalised fp32 partials and their LSE): the 8K MHA shape
    (P = 4 partials of [1, 8, 2048, 128]) and the 128K GQA shape (P = 8
    partials of [1, 32, 16384, 128], 2 GiB).  GB/s over the bytes read and
    written."""
    dev = torch.device("cuda")
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    stream = torch.cuda.current_stream()
    res = []
    for key in ("causal_mha_8k", "causal_gqa_128k"):
        wl = workload(key)
        L = wl.n // wl.P
        g = torch.Generator(device=dev).manual_seed(wl.seed + 7 + 1000 * rank)
        o = torch.randn((wl.P, wl.B, wl.Hq, L, wl.d_v), device=dev, generator=g)
        l = torch.randn((wl.P, wl.B, wl.Hq, L), device=dev, generator=g) * 3
        out = torch.empty((wl.B, wl.Hq, L, wl.d_v), device=dev, dtype=wl.torch_dtype)
        lse = torch.empty((wl.B, wl.Hq, L), device=dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        for _ in range(3):
            ra.lse_merge(o, l, wl.torch_dtype, out, lse)
        steps = max(3, min(args.steps, 10))
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ra.lse_merge(o, l, wl.torch_dtype, out, lse)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        assert ra.get_status() == ra.RA_OK
        ms = max_over_ranks(statistics.mean(ts), world)
        nbytes = (o.numel() + l.numel()) * 4 + out.numel() * out.element_size() + lse.numel() * 4
        gbs = nbytes / (ms * 1e-3) / 1e9
        res.append({"shape": f"{wl.name}: P={wl.P} partials of [{wl.B}, {wl.Hq}, {L}, {wl.d_v}]",
                    "value": round(world * gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
                    "bytes_per_step": nbytes,
                    "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                                 "unit": "GB/s", "frac": round(gbs / peak, 4),
                                 "peak_kind": f"{peaks_kind} HBM copy",
                                 "kernel": "lse_merge_few_kernel" if wl.P <= 4 else "lse_merge_kernel"}})
        del o, l, out, lse, flush
        torch.cuda.empty_cache()
    return res


def run_backward_leg(args, world, rank, wl, peaks, peaks_kind):
    """Gradients of the fused ring (dQ, dK, dV from the forward's O, LSE and a
    random dO) on workload `wl`: TFLOP/s of the whole backward call (row
    statistics, the tensor-core kernel, the dQ conversion), L2 flushed
    between steps."""
    from ring_context_parallelism_ra_b200.workloads import backward_flops, make_dout
    dev = torch.device("cuda")
    wr = dataclasses.replace(wl, seed=wl.seed + 1000 * rank)
    q, k, v = make_workload_inputs(wr, device=dev)
    g = make_dout(wl.B, wl.Hq, wl.n, wl.d_v, wl.torch_dtype, seed=wr.seed, device=dev)
    out, lse = ra.ring_forward(q, k, v, wl.P, wl.causal, wl.scale)
    ws = torch.empty(ra.backward_workspace_bytes(q, k, v), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ra.ring_backward(q, k, v, out, lse, g, wl.P, wl.causal, wl.scale, dq, dk, dv, ws)

    for _ in range(3):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    launches0 = ra.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for s, e in ev:
            flush.zero_()
            s.record(stream)
            step()
            e.record(stream)
        torch.cuda.synchronize()
    launches = ra.launch_count() - launches0
    assert ra.get_status() == ra.RA_OK
    ms_local = statistics.mean(s.elapsed_time(e) for s, e in ev)
    ms = max_over_ranks(ms_local, world)
    flops = backward_flops(wl)
    achieved = flops / (ms_local * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tr = load_traffic(f"ring_backward:{wl.name}", BWD192_FILES if wl.d_qk == 192 else BWD_FILES)
    del q, k, v, g, out, lse, ws, dq, dk, dv, flush
    torch.cuda.empty_cache()
    return {"workload": wl.name, "value": round(world * flops / (ms * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "flops_per_step": flops,
            "flop_convention": "2*B*Hq*n^2*(3*d_qk+2*d_v), x1/2 causal",
            "launches_per_step": launches // steps,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "peak_kind": f"{peaks_kind} bf16 burst",
                         "frac_of_sustained": round(
                             achieved / peaks.get("bf16_tflops_sustained", 1400.0), 4),
                         "traffic": tr["dram_bytes_per_launch"] if tr else None,
                         "traffic_kernel": ("bwd_tc192_kernel" if wl.d_qk == 192 else "bwd_tc_kernel")
                                           + " (ncu capture)",
                         "kernel": "ring_backward (prep + tcgen05 kernel + dQ conversion)"},
            "clocks": clk.summary()}


TC_FILES = ["tc_attention.cu", "item_queue.cuh", "ptx.cuh", "block_class.cuh"]
# every prefill workload is timed: the headline one in the main leg, the
# others in the `workloads` leg
PREFILL_WORKLOADS = ("causal_mla_256k", "causal_gqa_128k", "causal_mha_8k", "noncausal_fp32_512")
# the backward leg (every bf16 prefill workload; all run on the tensor cores)
BACKWARD_WORKLOADS = ("causal_mla_256k", "causal_gqa_128k", "causal_mha_8k")
BWD_FILES = ["bwd_attention.cu", "bwd_tc.cuh", "item_queue.cuh", "bwd.cuh", "ptx.cuh", "block_class.cuh"]
BWD192_FILES = ["bwd_tc192.cu", "bwd_tc.cuh", "item_queue.cuh", "bwd.cuh", "ptx.cuh", "block_class.cuh"]


def run_striped_leg(args, world, rank, wl, peaks):
    """Striped split (token p in partition p mod P) on workload `wl` (the
    causal GQA 128K workload, P = 8, where one partition block alone fills
    the GPU, so a block's time tracks its work):
    (a) the fused striped ring vs the fused contiguous ring, TFLOP/s;
    (b) P devices emulated one after another: device i runs its ring steps as
        block partials (Q_i against each KV_j it must see), timed as one chain
        of launches; the slowest device bounds a real ring's time.  Contiguous
        devices skip their fully masked blocks, striped devices have none."""
    from ring_context_parallelism_ra_b200.workloads import striped_order
    dev = torch.device("cuda")
    q, k, v = make_workload_inputs(dataclasses.replace(wl, seed=wl.seed + 1000 * rank), device=dev)
    flops = prefill_flops(wl)
    n, P, L = wl.n, wl.P, wl.n // wl.P
    order = torch.tensor(striped_order(n, P), device=dev)
    qs, ks, vs = (x[:, :, order].contiguous() for x in (q, k, v))
    out = torch.empty((wl.B, wl.Hq, n, wl.d_v), device=dev, dtype=wl.torch_dtype)
    lse = torch.empty((wl.B, wl.Hq, n), device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    steps = 3

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    ms_striped = timed(lambda: ra.ring_forward_striped(qs, ks, vs, P, wl.causal, wl.scale, out, lse))
    ms_contig = timed(lambda: ra.ring_forward(q, k, v, P, wl.causal, wl.scale, out, lse))
    # T(cp = 1): the whole sequence as one partition on this one device
    ms_one = timed(lambda: ra.ring_forward(q, k, v, 1, wl.causal, wl.scale, out, lse))
    parts = {}
    for name, (qq, kk, vv) in (("contiguous", (q, k, v)), ("striped", (qs, ks, vs))):
        qi = [qq[:, :, i * L:(i + 1) * L].contiguous() for i in range(P)]
        kj = [kk[:, :, j * L:(j + 1) * L].contiguous() for j in range(P)]
        vj = [vv[:, :, j * L:(j + 1) * L].contiguous() for j in range(P)]
        o = torch.empty((wl.B, wl.Hq, L, wl.d_v), device=dev)
        ll = torch.empty((wl.B, wl.Hq, L), device=dev)
        per_dev = []
        for i in range(P):
            if name == "contiguous":
                blocks = [(j, i * L, j * L, 1) for j in range(P) if not (wl.causal and j > i)]
            else:
                blocks = [(j, i, j, P) for j in range(P)]

            def chain(blocks=blocks, i=i):
                for j, qo, ko, st in blocks:
                    ra.block_partial_strided(qi[i], kj[j], vj[j], qo, ko, st, wl.causal, wl.scale, o, ll)
            per_dev.append(timed(chain))
        parts[name] = per_dev
    assert ra.get_status() == ra.RA_OK
    res = {"workload": wl.name,
           "fused_striped_tflops": round(flops / (ms_striped * 1e-3) / 1e12, 2),
           "fused_contiguous_tflops": round(flops / (ms_contig * 1e-3) / 1e12, 2),
           "emulated_devices": P,
           "device_ms_contiguous": [round(x, 4) for x in parts["contiguous"]],
           "device_ms_striped": [round(x, 4) for x in parts["striped"]],
           "slowest_device_ms": {k: round(max(v), 4) for k, v in parts.items()},
           "ring_speedup_striped_over_contiguous":
               round(max(parts["contiguous"]) / max(parts["striped"]), 3),
           # scaling efficiency eta(cp) = T(cp = 1) / (cp T(cp)), T(cp) = the
           # slowest emulated device (the exchange, hidden under the blocks on
           # NVLink, and the final merge are not in it)
           "t_cp1_ms": round(ms_one, 4),
           "eta_cp": {k: round(ms_one / (P * max(v)), 4) for k, v in parts.items()},
           "note": "block partials per emulated device, one device at a time on this GPU"}
    del q, k, v, qs, ks, vs, out, lse, flush
    torch.cuda.empty_cache()
    return res


def short_cache_decode_latency(wl, world, tokens=32768, reps=50):
    """Latency of one pass-Q decode step on a short cache (same heads and
    shards as `wl`): issued call by call, and replayed as one captured CUDA
    graph (host_pipeline.PassQDecodeGraph).  Wall time of `reps` back-to-back
    steps per mode, divided by `reps` (host enqueue cost included)."""
    from ring_context_parallelism_ra_b200.host_pipeline import PassQDecodeGraph
    from ring_context_parallelism_ra_b200.workloads import make_qkv
    dev = torch.device("cuda")
    q, k, v = make_qkv(wl.B, wl.Hq, wl.Hkv, 1, tokens, wl.d_qk, wl.d_v, wl.torch_dtype,
                       seed=wl.seed + 5, device=dev)
    graph = PassQDecodeGraph(k, v, wl.P, wl.Hq, wl.scale)
    graph.q.copy_(q)
    bufs = graph.bufs

    def timed(step):
        for _ in range(5):
            step()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            step()
        e1.record()
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / reps, world) * 1e3

    eager_us = timed(lambda: ra.decode_pass_q(graph.q, k, v, wl.P, wl.scale, bufs))
    graph_us = timed(graph.replay)
    # for scale: the same cache as ONE shard (one chunk-kernel launch over
    # every chunk plus its chunk merge), what a single device would run
    ws1 = torch.empty(ra.decode_workspace_bytes(wl.B, wl.Hq, wl.Hkv, tokens), dtype=torch.uint8,
                      device=dev)
    o1 = torch.empty((wl.B, wl.Hq, wl.d_v), device=dev)
    l1 = torch.empty((wl.B, wl.Hq), device=dev)
    one_us = timed(lambda: ra.decode_partial(graph.q, k, v, 0, tokens, wl.scale, ws1, o1, l1))
    assert ra.get_status() == ra.RA_OK
    kv_bytes = 2 * wl.B * wl.Hkv * tokens * wl.d_qk * 2
    del graph, q, k, v, ws1, o1, l1
    torch.cuda.empty_cache()
    return {"tokens": tokens, "shards": wl.P,
            "launches_per_step": 3 if (tokens // wl.P) % 2048 == 0 else 2 * wl.P + 1,
            "eager_us_per_step": round(eager_us, 2), "graph_us_per_step": round(graph_us, 2),
            "one_shard_us_per_step": round(one_us, 2), "kv_bytes": kv_bytes}


def run_decode_leg(args, world, rank, peaks, peaks_kind):
    """Pass-Q decode over the 1M-token cache (P shards + merge): GB/s of K/V read."""
    wl = workload("decode_1m")
    dev = torch.device("cuda")
    q, k, v = make_workload_inputs(wl, device=dev)
    P = wl.P
    L = wl.n // P
    ws = torch.empty(ra.decode_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.n), dtype=torch.uint8,
                     device=dev)  # every chunk of every shard (ra_decode_partials)
    o_parts = torch.empty((P, wl.B, wl.Hq, wl.d_v), device=dev)
    l_parts = torch.empty((P, wl.B, wl.Hq), device=dev)
    out = torch.empty((wl.B, wl.Hq, wl.d_v), device=dev, dtype=wl.torch_dtype)
    lse = torch.empty((wl.B, wl.Hq), device=dev)
    bufs = {"o_parts": o_parts, "lse_parts": l_parts, "workspace": ws, "out": out, "lse": lse}
    stream = torch.cuda.current_stream()
    for _ in range(3):
        ra.decode_pass_q(q, k, v, P, wl.scale, bufs)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for s, e in ev:
            s.record(stream)
            ra.decode_pass_q(q, k, v, P, wl.scale, bufs)
            e.record(stream)
        torch.cuda.synchronize()
    assert ra.get_status() == ra.RA_OK
    ms_local = statistics.mean(s.elapsed_time(e) for s, e in ev)
    ms = max_over_ranks(ms_local, world)
    nbytes = decode_kv_bytes(wl)
    gbs = nbytes / (ms_local * 1e-3) / 1e9
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    del q, k, v, ws
    torch.cuda.empty_cache()
    short = short_cache_decode_latency(wl, world)
    return {"workload": wl.name, "short_cache": short,
            "value": round(world * nbytes / (ms * 1e-3) / 1e9, 1),
            "unit": "GB/s", "ms_per_step": round(ms, 4), "bytes_per_step": nbytes,
            "launches_per_step": 3 if L % 2048 == 0 else 2 * P + 1, "kv_bytes_exceed_l2": True,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "peak_kind": f"{peaks_kind} HBM copy",
                         "kernel": "decode pass-Q (chunk kernel + two merges)"},
            "clocks": clk.summary()}


# -------------------------------------------------------- reference arm ----

def run_reference(args, world, rank):
    wl = workload(args.workload)
    budget = float(os.environ.get("RA_ORACLE_BUDGET_S", "12"))
    vals, walls = [], []
    desc, cores = "", 0
    for i in range(args.warmup + args.steps):
        per = budget / max(1, args.steps) if i >= args.warmup else min(2.0, budget / 10)
        val, cores, desc, dt = oracle_sample(wl, per, seed=i)
        if i >= args.warmup:
            vals.append(val)
            walls.append(dt)
    value = statistics.mean(vals)
    flops = prefill_flops(wl)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        # each step is a bounded sample of the workload: its measured wall time
        "ms_per_step": round(statistics.mean(walls) * 1e3, 3),
        "ms_per_step_full_workload_extrapolated": round(flops / (value * 1e12) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_of(wl, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": desc + " per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="causal_mla_256k",
                    choices=["causal_mha_8k", "causal_gqa_128k", "causal_mla_256k",
                             "noncausal_fp32_512"])
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-striped", action="store_true")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--skip-merge", action="store_true")
    ap.add_argument("--skip-workloads", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks do nothing
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps(run_reference(args, world, 0)), flush=True)
        return
    world, rank, _ = dist_setup(args.gpus)
    line = run_ours(args, world, rank)
    if rank == 0:
        val, cores, desc, _ = oracle_sample(workload(args.workload), args.cpu_budget_s)
        line["cpu_baseline"] = {"value": round(val, 6), "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle", "sample": desc}
        line["recap"] = recap(line)
        for key in ("decode_short_cache", "decode"):   # keep the decode leg last
            if key in line:
                line[key] = line.pop(key)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
