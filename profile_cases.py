"""Small, fixed launches of each kernel for profiler captures.

    python profile_cases.py CASE [--reps N]

Each case runs two warm-up launches and then N (default 1) launches of one
kernel at a shape the bench uses, holding at most a few GB on the device
(``--activity``: the same launches recorded by torch.profiler, each
kernel's device time printed; no replay, unlike ncu):

  prefill_mha8k   fused ring forward, causal MHA, 8 heads, n = 8192, d = 128,
                 P = 4 (the bench's default workload, one launch per step)
  prefill_gqa32k fused ring forward, causal GQA 32/8 heads, n = 32768, P = 8
  prefill_mla32k fused ring forward, causal MLA-shaped head (d_qk = 192,
                 d_v = 128), 16 heads, n = 32768, P = 16 (the 256K workload's
                 head shape and partition count at an eighth of its length)
  prefill_mla256k / prefill_gqa128k
                 fused ring forward on the full 256K MLA / 128K GQA workloads
                 (what the bench times; for single-pass counters only)
  backward_mla256k / backward_gqa128k
                 ring backward on the same full-size workloads
  backward_mla32k ring backward, the MLA-shaped head at n = 32768 (as
                 prefill_mla32k)
  decode_shard   pass-Q decode partial on one 131072-token shard of the
                 1M-token cache (B = 4, 64/8 heads): one chunk-kernel launch
                 and one merge launch, as one shard of the bench's decode step
  merge_p8       LSE merge of 8 fp32 partials of shape [1, 32, 16384, 128]
  merge_p4_8k    LSE merge of 4 fp32 partials of shape [1, 8, 2048, 128] (the
                 partials one query partition of the 8K MHA ring collects)
  backward_mha8k  ring backward (prep, tensor-core kernel, dQ conversion) on the
                 bench's default workload, from its own forward O and LSE
  backward_gqa32k ring backward, causal GQA 32/8 heads, n = 32768, P = 8
"""
from __future__ import annotations

import argparse

import torch

import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from ring_context_parallelism_ra_b200 import ra  # noqa: E402
from ring_context_parallelism_ra_b200.workloads import (make_dout, make_qkv,  # noqa: E402
                                                        make_workload_inputs, workload)


# With --activity every launch starts from a cold L2, as in the bench: a
# 256 MiB buffer is written before it.
_FLUSH = {"on": False, "buf": None}


def _flush():
    if _FLUSH["on"]:
        if _FLUSH["buf"] is None:
            _FLUSH["buf"] = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        _FLUSH["buf"].zero_()


def _prefill(q, k, v, P, reps):
    out = torch.empty((*q.shape[:3], v.shape[-1]), device=q.device, dtype=q.dtype)
    lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
    for _ in range(2 + reps):
        _flush()
        ra.ring_forward(q, k, v, P, True, None, out, lse)
    torch.cuda.synchronize()


def _backward(q, k, v, P, reps):
    g = make_dout(q.shape[0], q.shape[1], q.shape[2], v.shape[-1], q.dtype, seed=9, device=q.device)
    out, lse = ra.ring_forward(q, k, v, P, True)
    ws = torch.empty(ra.backward_workspace_bytes(q, k, v), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for _ in range(2 + reps):
        _flush()
        ra.ring_backward(q, k, v, out, lse, g, P, True, None, dq, dk, dv, ws)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["prefill_mha8k", "prefill_gqa32k", "prefill_mla32k",
                                     "prefill_mla256k", "prefill_gqa128k", "backward_mla256k",
                                     "backward_gqa128k", "backward_mla32k", "decode_shard",
                                     "merge_p8",
                                     "merge_p4_8k", "backward_mha8k", "backward_gqa32k"])
    ap.add_argument("--reps", type=int, default=1)
    ap.add_argument("--activity", action="store_true",
                    help="record the launches with torch.profiler (kernel activity records, "
                         "no replay) and print each kernel's device time")
    args = ap.parse_args()
    if args.activity:
        from torch.profiler import ProfilerActivity, profile
        _FLUSH["on"] = True
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            run_case(args)
        print(prof.key_averages().table(sort_by="cuda_time_total", row_limit=12,
                                        max_name_column_width=70))
    else:
        run_case(args)
    assert ra.get_status() == ra.RA_OK
    print(f"{args.case}: ok")


def run_case(args):
    dev = "cuda"
    if args.case == "prefill_mha8k":
        wl = workload("causal_mha_8k")
        q, k, v = make_workload_inputs(wl, device=dev)
        _prefill(q, k, v, wl.P, args.reps)
    elif args.case == "prefill_gqa32k":
        q, k, v = make_qkv(1, 32, 8, 32768, 32768, 128, 128, torch.bfloat16, seed=3, device=dev)
        _prefill(q, k, v, 8, args.reps)
    elif args.case == "prefill_mla32k":
        q, k, v = make_qkv(1, 16, 16, 32768, 32768, 192, 128, torch.bfloat16, seed=5, device=dev)
        _prefill(q, k, v, 16, args.reps)
    elif args.case in ("prefill_mla256k", "prefill_gqa128k"):
        wl = workload("causal_mla_256k" if args.case == "prefill_mla256k" else "causal_gqa_128k")
        q, k, v = make_workload_inputs(wl, device=dev)
        _prefill(q, k, v, wl.P, args.reps)
    elif args.case in ("backward_mla256k", "backward_gqa128k"):
        wl = workload("causal_mla_256k" if args.case == "backward_mla256k" else "causal_gqa_128k")
        q, k, v = make_workload_inputs(wl, device=dev)
        _backward(q, k, v, wl.P, args.reps)
    elif args.case == "backward_mla32k":
        q, k, v = make_qkv(1, 16, 16, 32768, 32768, 192, 128, torch.bfloat16, seed=5, device=dev)
        _backward(q, k, v, 16, args.reps)
    elif args.case == "backward_mha8k":
        wl = workload("causal_mha_8k")
        q, k, v = make_workload_inputs(wl, device=dev)
        _backward(q, k, v, wl.P, args.reps)
    elif args.case == "backward_gqa32k":
        q, k, v = make_qkv(1, 32, 8, 32768, 32768, 128, 128, torch.bfloat16, seed=3, device=dev)
        _backward(q, k, v, 8, args.reps)
    elif args.case == "decode_shard":
        q, k, v = make_qkv(4, 64, 8, 1, 131072, 128, 128, torch.bfloat16, seed=4, device=dev)
        ws = torch.empty(ra.decode_workspace_bytes(4, 64, 8, 131072), dtype=torch.uint8, device=dev)
        o = torch.empty((4, 64, 128), device=dev)
        l = torch.empty((4, 64), device=dev)
        for _ in range(2 + args.reps):
            ra.decode_partial(q, k, v, 0, 131072, None, ws, o, l)
        torch.cuda.synchronize()
    else:
        P, H, L = (8, 32, 16384) if args.case == "merge_p8" else (4, 8, 2048)
        g = torch.Generator(device=dev).manual_seed(5)
        o = torch.randn((P, 1, H, L, 128), device=dev, generator=g)
        l = torch.randn((P, 1, H, L), device=dev, generator=g)
        out = torch.empty((1, H, L, 128), device=dev, dtype=torch.bfloat16)
        lse = torch.empty((1, H, L), device=dev)
        for _ in range(2 + args.reps):
            _flush()
            ra.lse_merge(o, l, torch.bfloat16, out, lse)
        torch.cuda.synchronize()


if __name__ == "__main__":
    main()
