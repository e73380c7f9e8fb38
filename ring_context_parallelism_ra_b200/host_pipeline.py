"""Host-side drivers of the library's calls: the fused ring forward over a
stream of host-resident batches (``RingForwardPipeline``), and a pass-Q
decode step captured once as a CUDA graph (``PassQDecodeGraph``).

RingForwardPipeline: the copies of one batch overlap the computation of its
neighbours.

Each batch goes host -> device (pinned memory, copy stream), through
``ra.ring_forward`` (compute stream) and its output and LSE back to pinned
host memory (a second copy stream).  Two device buffer sets alternate, so
batch i + 1's inputs travel while batch i computes and batch i - 1's results
return.  This is host-side plumbing only: the attention runs in the
library's kernel, the copies are plain ``cudaMemcpyAsync`` through torch.
"""
from __future__ import annotations

import torch

from . import ra

__all__ = ["RingForwardPipeline", "PassQDecodeGraph"]


class RingForwardPipeline:
    """``submit`` host batches (q, k, v pinned CPU tensors of one shape), get
    each batch's (O, LSE) in pinned host memory once ``wait`` has returned
    for it.  Results of batch i live in slot i % depth and are overwritten by
    batch i + depth."""

    def __init__(self, q_shape, k_shape, v_shape, dtype, P, causal=True, scale=None,
                 device="cuda", depth=2):
        self.P, self.causal, self.scale, self.depth = P, causal, scale, depth
        B, Hq, n, _ = q_shape
        dv = v_shape[-1]
        self.dev = [{"q": torch.empty(q_shape, dtype=dtype, device=device),
                     "k": torch.empty(k_shape, dtype=dtype, device=device),
                     "v": torch.empty(v_shape, dtype=dtype, device=device),
                     "out": torch.empty((B, Hq, n, dv), dtype=dtype, device=device),
                     "lse": torch.empty((B, Hq, n), dtype=torch.float32, device=device)}
                    for _ in range(depth)]
        self.host = [{"out": torch.empty((B, Hq, n, dv), dtype=dtype, pin_memory=True),
                      "lse": torch.empty((B, Hq, n), dtype=torch.float32, pin_memory=True)}
                     for _ in range(depth)]
        self.s_in = torch.cuda.Stream(device=device)
        self.s_comp = torch.cuda.Stream(device=device)
        self.s_out = torch.cuda.Stream(device=device)
        mk = lambda: [torch.cuda.Event() for _ in range(depth)]  # noqa: E731
        self.in_done, self.comp_done, self.out_done = mk(), mk(), mk()
        self.used = [False] * depth
        self.count = 0

    def submit(self, q, k, v):
        """Enqueue one batch; returns its slot index."""
        slot = self.count % self.depth
        d, h = self.dev[slot], self.host[slot]
        with torch.cuda.stream(self.s_in):
            if self.used[slot]:  # the slot's inputs were read by its previous kernel
                self.s_in.wait_event(self.comp_done[slot])
            d["q"].copy_(q, non_blocking=True)
            d["k"].copy_(k, non_blocking=True)
            d["v"].copy_(v, non_blocking=True)
            self.in_done[slot].record(self.s_in)
        with torch.cuda.stream(self.s_comp):
            self.s_comp.wait_event(self.in_done[slot])
            if self.used[slot]:  # the slot's outputs have left for the host
                self.s_comp.wait_event(self.out_done[slot])
            ra.ring_forward(d["q"], d["k"], d["v"], self.P, self.causal, self.scale, d["out"],
                            d["lse"], stream=self.s_comp)
            self.comp_done[slot].record(self.s_comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.comp_done[slot])
            h["out"].copy_(d["out"], non_blocking=True)
            h["lse"].copy_(d["lse"], non_blocking=True)
            self.out_done[slot].record(self.s_out)
        self.used[slot] = True
        self.count += 1
        return slot

    def wait(self, slot):
        """Block until the slot's latest results are in host memory; return them."""
        self.out_done[slot].synchronize()
        return self.host[slot]["out"], self.host[slot]["lse"]

    def drain_on(self, stream):
        """Make `stream` wait for everything submitted so far."""
        for s in range(self.depth):
            if self.used[s]:
                stream.wait_event(self.out_done[s])


class PassQDecodeGraph:
    """Pass-Q decode over a fixed KV cache, captured once as a CUDA graph.

    A decode step is P shard partials and their merge: with a short cache
    every launch is short, and the CP study (page "上下文并行 (CP) 收益评估实验
    设计", decode section) calls this step latency-bound.  Replaying the
    captured graph enqueues the whole step at once.  Write the new query
    token into ``q`` (a static device buffer [B, Hq, 1, d]) before each
    ``replay``; the cache tensors must stay at their addresses.  ``out`` and
    ``lse`` hold the result after the replay has run on the stream.
    """

    def __init__(self, k, v, P, Hq, scale=None, stream=None):
        B, Hkv, S, d = k.shape
        if S % P:
            raise ValueError("cache length must split into P equal shards")
        dev = k.device
        self.k, self.v, self.P, self.scale = k, v, P, scale
        self.q = torch.zeros((B, Hq, 1, d), device=dev, dtype=k.dtype)
        self.bufs = {
            "o_parts": torch.empty((P, B, Hq, v.shape[-1]), device=dev, dtype=torch.float32),
            "lse_parts": torch.empty((P, B, Hq), device=dev, dtype=torch.float32),
            "workspace": torch.empty(ra.decode_workspace_bytes(B, Hq, Hkv, S),
                                     dtype=torch.uint8, device=dev),
            "out": torch.empty((B, Hq, v.shape[-1]), device=dev, dtype=k.dtype),
            "lse": torch.empty((B, Hq), device=dev, dtype=torch.float32),
        }
        self.out, self.lse = self.bufs["out"], self.bufs["lse"]
        self.stream = stream if stream is not None else torch.cuda.Stream(device=dev)
        # one eager run first: the library sets up its per-device state
        # (status word, kernel attributes) outside the capture
        with torch.cuda.stream(self.stream):
            self._step()
        self.stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            self._step()

    def _step(self):
        ra.decode_pass_q(self.q, self.k, self.v, self.P, self.scale, self.bufs)

    def replay(self):
        """Enqueue one decode step; returns (out [B, Hq, d_v], lse [B, Hq])."""
        self.graph.replay()
        return self.out, self.lse
