"""Ring Attention across devices: one sequence partition per rank, the KV
partitions passed around the ring.

Method (pages cited by title and section): each device keeps its query
partition Q_i and sends its KV partition to the next device while receiving
the previous device's, so that after P - 1 exchanges every query partition
has met every KV partition (page "AI 推理系列（十一）：Ring Attention 如何让
多张 GPU 共同计算一条超长序列", section "KV 在 Ring 中如何流动"); the exchange of
step s + 1 overlaps the block computation of step s (same page, section "通信
很多，为什么仍然可能划算"; page "LLM长文本推理Ring Attention环形注意力机制实现与
优化", section "Ring Attention实现代码与通信重叠").  Each block partial is folded
into a running (O, LSE) with the log-sum-exp rule as soon as it is computed
(the latter page's per-step update), so a rank holds two partials, not P.  With a causal mask a contiguous
split skips the blocks wholly in the future (and leaves the devices unevenly
loaded); the striped split of the latter page's tuning section gives rank r
the tokens r, r + P, r + 2P, ... so that every block is about half visible.

Backward: KV_j travels together with its gradient accumulators dK_j, dV_j,
which collect one share per query partition; dQ_i collects at its rank; a
last hop returns every accumulator to its owner.  A rank computes its share
of step s into a local buffer while the accumulator it must add it to is
still on its way from the previous rank, then adds the two and sends the sum
on: the accumulator hop overlaps the block computation instead of
following it.

Layout on every rank: q [B, Hq, L, d_qk], k [B, Hkv, L, d_qk], v [B, Hkv, L,
d_v] with L = n / P tokens of its partition, in position order.  Rank r is
partition r of the ring (ring order = rank order of the process group).

Transports:
  * ``NcclTransport`` -- device tensors exchanged with batched NCCL
    send / recv; the process group's side stream runs the exchange while the
    current stream runs the block kernel.
  * ``HostTransport`` -- send / recv through host memory (a gloo process
    group, or CPU tensors); the exchange is synchronous.

Ulysses (page "AI 推理系列（十一）…", section "Ring 与 Ulysses：同样切序列，通信
方式不同"): the same token partitions are re-sharded before attention by an
all-to-all of Q, K, V so that every device holds a share of the heads over
the whole sequence, attends locally, and a second all-to-all restores the
sequence layout.  ``ulysses_attention_forward`` / ``_backward`` implement it
with the library's single-device kernels for the local attention; the head
count must split evenly over the devices (H_q % P == H_kv % P == 0).

Pass-Q decode (page "上下文并行 (CP) 收益评估实验设计", decode section and the
pass-KV / pass-Q term): the KV cache is split by token range, one shard per
device; the single query token of each sequence goes to every device, each
device computes the normalised partial attention of the query over its own
shard, and the partials are reduced.  ``pass_q_decode`` sends the query from
one rank, gathers every rank's (O_p, LSE_p) in one collective, and merges
them with the log-sum-exp rule on every rank, so all ranks return the same
result.

The block arithmetic is a pluggable ``blocks`` object; ``KernelBlocks`` (the
default) runs the library's CUDA kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ra

__all__ = ["KernelBlocks", "NcclTransport", "HostTransport", "default_transport",
           "ring_attention_forward", "ring_attention_backward", "partition_positions",
           "ulysses_attention_forward", "ulysses_attention_backward", "pass_q_decode"]


class KernelBlocks:
    """Block arithmetic on the library's kernels (bf16 on tensor cores, fp32
    exact)."""

    def partial(self, q, k, v, q_offset, k_offset, stride, causal, scale, o, lse):
        return ra.block_partial_strided(q, k, v, q_offset, k_offset, stride, causal, scale, o, lse)

    def merge(self, o_parts, lse_parts, out_dtype, out=None, lse=None):
        return ra.lse_merge(o_parts, lse_parts, out_dtype, out, lse)

    def delta(self, out, dout):
        return ra.backward_delta(out, dout)

    def backward(self, q, k, v, dout, lse, delta, q_offset, k_offset, stride, causal, scale,
                 dq_acc, dk_acc, dv_acc):
        ra.block_backward(q, k, v, dout, lse, delta, q_offset, k_offset, stride, causal, scale,
                          dq_acc, dk_acc, dv_acc)

    def full(self, q, k, v, causal, scale):
        return ra.ring_forward(q, k, v, 1, causal, scale)

    def full_backward(self, q, k, v, out, lse, dout, causal, scale):
        return ra.ring_backward(q, k, v, out, lse, dout, 1, causal, scale)

    def decode_partial(self, q, k, v, scale, o_part, lse_part):
        ra.decode_partial(q, k, v, scale=scale, o_part=o_part, lse_part=lse_part)

    def decode_merge(self, o_parts, lse_parts, out_dtype):
        return ra.decode_merge(o_parts, lse_parts, out_dtype)


class _Done:
    def wait(self):
        return None


def _peer(group, r):
    """Global rank of rank `r` of `group` (point-to-point calls take global ranks)."""
    return r if group is None else dist.get_global_rank(group, r)


class NcclTransport:
    """Send to the next rank and receive from the previous one with batched
    NCCL point-to-point operations (asynchronous)."""

    def __init__(self, group=None):
        self.group = group

    def exchange(self, send, recv, nxt, prv):
        nxt, prv = _peer(self.group, nxt), _peer(self.group, prv)
        ops = [dist.P2POp(dist.isend, t, nxt, self.group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, prv, self.group) for t in recv]
        reqs = dist.batch_isend_irecv(ops)

        class _Handle:
            def wait(self_inner):
                for r in reqs:
                    r.wait()
        return _Handle()

    def all_to_all(self, send, recv):
        """send[c] goes to rank c, recv[c] comes from rank c (device tensors)."""
        dist.all_to_all(recv, send, group=self.group)

    def broadcast(self, t, src):
        """Overwrite `t` on every rank with rank `src`'s `t`."""
        dist.broadcast(t, _peer(self.group, src), group=self.group)

    def all_gather(self, out, inp):
        """out[c] = rank c's `inp` (out: [P, *inp.shape], contiguous)."""
        dist.all_gather_into_tensor(out, inp, group=self.group)


class HostTransport:
    """Send / recv through host memory (for a gloo process group).  Device
    tensors are staged through CPU copies; the exchange completes before
    ``exchange`` returns."""

    def __init__(self, group=None):
        self.group = group

    def exchange(self, send, recv, nxt, prv):
        me = dist.get_rank(self.group)
        nxt, prv = _peer(self.group, nxt), _peer(self.group, prv)
        staged = [t.detach().to("cpu") for t in send]
        bufs = [torch.empty(t.shape, dtype=t.dtype) for t in recv]
        # even ranks send first, odd ranks receive first: no cycle of blocking sends
        for t, b in zip(staged, bufs):
            if me % 2 == 0:
                dist.send(t, nxt, self.group)
                dist.recv(b, prv, self.group)
            else:
                dist.recv(b, prv, self.group)
                dist.send(t, nxt, self.group)
        for b, t in zip(bufs, recv):
            t.copy_(b)
        return _Done()

    def all_to_all(self, send, recv):
        """send[c] goes to rank c, recv[c] comes from rank c; completes before
        returning."""
        me = dist.get_rank(self.group)
        staged = [t.detach().to("cpu").contiguous() for t in send]
        bufs = [torch.empty(t.shape, dtype=t.dtype) for t in recv]
        bufs[me].copy_(staged[me])
        reqs = []
        for c in range(len(send)):
            if c != me:
                peer = _peer(self.group, c)
                reqs.append(dist.isend(staged[c], peer, self.group))
                reqs.append(dist.irecv(bufs[c], peer, self.group))
        for r in reqs:
            r.wait()
        for b, t in zip(bufs, recv):
            t.copy_(b)

    def broadcast(self, t, src):
        """Overwrite `t` on every rank with rank `src`'s `t`; completes before
        returning."""
        staged = t.detach().to("cpu").contiguous()
        dist.broadcast(staged, _peer(self.group, src), group=self.group)
        t.copy_(staged)

    def all_gather(self, out, inp):
        """out[c] = rank c's `inp`; completes before returning."""
        staged = inp.detach().to("cpu").contiguous()
        bufs = [torch.empty(staged.shape, dtype=staged.dtype) for _ in range(out.shape[0])]
        dist.all_gather(bufs, staged, group=self.group)
        out.copy_(torch.stack(bufs))


def default_transport(group=None):
    """NCCL for an NCCL process group, host staging otherwise."""
    backend = dist.get_backend(group)
    return NcclTransport(group) if backend == "nccl" else HostTransport(group)


def partition_positions(rank: int, P: int, L: int, striped: bool):
    """(offset, stride) of partition `rank`: token of local row t is
    offset + t * stride."""
    return (rank, P) if striped else (rank * L, 1)


def _ring_check(q, k, v):
    """The ring assumes one equal partition per rank: Q, K and V of a rank
    hold the same tokens."""
    if not (q.shape[2] == k.shape[2] == v.shape[2]) or q.shape[0] != k.shape[0] or \
            k.shape[:3] != v.shape[:3] or q.shape[-1] != k.shape[-1] or q.shape[1] % k.shape[1]:
        raise ValueError(f"ring partitions disagree: q {tuple(q.shape)}, k {tuple(k.shape)}, "
                         f"v {tuple(v.shape)}")


def _ring(group):
    P = dist.get_world_size(group)
    i = dist.get_rank(group)
    return P, i, (i + 1) % P, (i - 1) % P


def ring_attention_forward(q, k, v, causal=True, scale=None, striped=False, group=None,
                           transport=None, blocks=None):
    """This rank's output (O_i [B, Hq, L, d_v] in q's dtype, LSE_i fp32
    [B, Hq, L]) of exact attention over the whole sequence, its query
    partition meeting every KV partition as they pass around the ring."""
    _ring_check(q, k, v)
    P, i, nxt, prv = _ring(group)
    transport = transport or default_transport(group)
    blocks = blocks or KernelBlocks()
    B, Hq, L, _ = q.shape
    dv = v.shape[-1]
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    # the steps whose block is computed (a contiguous causal split skips the
    # blocks wholly in the future)
    todo = [s for s in range(P) if not (causal and not striped and (i - s) % P > i)]
    # running (O, LSE): slot 0 of a stack holds it, slot 1 the new block
    # partial; the merge writes the next running value into the other stack
    o_st = [torch.empty((2, B, Hq, L, dv), device=q.device, dtype=torch.float32)
            for _ in range(2 if len(todo) > 1 else 1)]
    l_st = [torch.empty((2, B, Hq, L), device=q.device, dtype=torch.float32) for _ in o_st]
    cur = [k.contiguous(), v.contiguous()]
    nbuf = [torch.empty_like(cur[0]), torch.empty_like(cur[1])]
    q_off, stride = partition_positions(i, P, L, striped)
    run, done, result = 0, 0, None
    for s in range(P):
        j = (i - s) % P
        handle = transport.exchange(cur, nbuf, nxt, prv) if s < P - 1 else _Done()
        k_off, _ = partition_positions(j, P, L, striped)
        if s in todo:
            slot = 0 if done == 0 else 1
            blocks.partial(q, cur[0], cur[1], q_off, k_off, stride, causal, scale,
                           o_st[run][slot], l_st[run][slot])
            done += 1
            if done == len(todo):     # the last fold writes the result itself
                n = 1 if done == 1 else 2
                result = blocks.merge(o_st[run][:n], l_st[run][:n], q.dtype)
            elif done > 1:
                blocks.merge(o_st[run], l_st[run], torch.float32, o_st[1 - run][0],
                             l_st[1 - run][0])
                run = 1 - run
        handle.wait()
        if s < P - 1:
            cur, nbuf = nbuf, cur
    return result


def ring_attention_backward(q, k, v, out, lse, dout, causal=True, scale=None, striped=False,
                            group=None, transport=None, blocks=None):
    """This rank's gradients (dQ_i, dK_i, dV_i, in q's dtype) of
    ``ring_attention_forward``; ``out`` and ``lse`` are its outputs here."""
    _ring_check(q, k, v)
    if out.shape[:3] != q.shape[:3] or dout.shape != out.shape or lse.shape != q.shape[:3]:
        raise ValueError("out, lse and dout must match this rank's query partition")
    P, i, nxt, prv = _ring(group)
    transport = transport or default_transport(group)
    blocks = blocks or KernelBlocks()
    B, Hq, L, _ = q.shape
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    delta = blocks.delta(out, dout)
    dq = torch.zeros(q.shape, device=q.device, dtype=torch.float32)
    kv = [k.contiguous(), v.contiguous()]
    kv_buf = [torch.empty_like(kv[0]), torch.empty_like(kv[1])]
    f32 = dict(device=q.device, dtype=torch.float32)
    share = [torch.empty(k.shape, **f32), torch.empty(v.shape, **f32)]   # this step's share
    acc_in = [torch.empty(k.shape, **f32), torch.empty(v.shape, **f32)]  # arriving accumulator
    acc_out = [torch.empty(k.shape, **f32), torch.empty(v.shape, **f32)]  # sum sent on
    q_off, stride = partition_positions(i, P, L, striped)
    for s in range(P):
        j = (i - s) % P
        # K, V of the next step travel while this step computes
        handle = transport.exchange(kv, kv_buf, nxt, prv) if s < P - 1 else _Done()
        # KV_j's accumulator arrives from the previous rank (which added its
        # share in its step s - 1) while this rank sends the sum of its step
        # s - 1; at s = 0 KV_j is this rank's own and starts from zero
        acc_h = transport.exchange(acc_out, acc_in, nxt, prv) if s > 0 else _Done()
        k_off, _ = partition_positions(j, P, L, striped)
        share[0].zero_()
        share[1].zero_()
        if not (causal and not striped and j > i):
            blocks.backward(q, kv[0], kv[1], dout, lse, delta, q_off, k_off, stride, causal,
                            scale, dq, share[0], share[1])
        acc_h.wait()
        if s > 0:
            torch.add(acc_in[0], share[0], out=acc_out[0])
            torch.add(acc_in[1], share[1], out=acc_out[1])
        else:
            acc_out[0].copy_(share[0])
            acc_out[1].copy_(share[1])
        handle.wait()
        if s < P - 1:
            kv, kv_buf = kv_buf, kv
    if P > 1:  # a last hop returns every accumulator to its owner
        transport.exchange(acc_out, acc_in, nxt, prv).wait()
        acc_out = acc_in
    return dq.to(q.dtype), acc_out[0].to(k.dtype), acc_out[1].to(v.dtype)


def _seq_to_heads(x, P, transport):
    """[B, H, L, d] sequence partition of every head -> [B, H / P, P * L, d]:
    this rank's head share over the whole sequence (partitions in rank
    order)."""
    B, H, L = x.shape[:3]
    hp = H // P
    send = [x[:, c * hp:(c + 1) * hp].contiguous() for c in range(P)]
    recv = [torch.empty_like(send[0]) for _ in range(P)]
    transport.all_to_all(send, recv)
    return torch.cat(recv, dim=2)


def _heads_to_seq(y, P, transport):
    """Inverse of ``_seq_to_heads``: [B, H / P, P * L, ...] -> [B, H, L, ...]."""
    L = y.shape[2] // P
    send = [y[:, :, c * L:(c + 1) * L].contiguous() for c in range(P)]
    recv = [torch.empty_like(send[0]) for _ in range(P)]
    transport.all_to_all(send, recv)
    return torch.cat(recv, dim=1)


def _ulysses_check(q, k, P):
    if q.shape[1] % P or k.shape[1] % P:
        raise ValueError(f"Ulysses needs H_q ({q.shape[1]}) and H_kv ({k.shape[1]}) divisible "
                         f"by the {P} devices")


def ulysses_attention_forward(q, k, v, causal=True, scale=None, group=None, transport=None,
                              blocks=None):
    """This rank's output (O_i [B, Hq, L, d_v], LSE_i [B, Hq, L]) of exact
    attention over the whole sequence; rank r holds the contiguous tokens
    [r L, (r + 1) L) of every head on entry and on return."""
    P = dist.get_world_size(group)
    transport = transport or default_transport(group)
    blocks = blocks or KernelBlocks()
    _ulysses_check(q, k, P)
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    qh, kh, vh = (_seq_to_heads(x, P, transport) for x in (q, k, v))
    o, lse = blocks.full(qh, kh, vh, causal, scale)
    return (_heads_to_seq(o, P, transport),
            _heads_to_seq(lse.unsqueeze(-1), P, transport)[..., 0].contiguous())


def ulysses_attention_backward(q, k, v, out, lse, dout, causal=True, scale=None, group=None,
                               transport=None, blocks=None):
    """This rank's gradients (dQ_i, dK_i, dV_i) of ``ulysses_attention_forward``."""
    P = dist.get_world_size(group)
    transport = transport or default_transport(group)
    blocks = blocks or KernelBlocks()
    _ulysses_check(q, k, P)
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    qh, kh, vh, oh, gh = (_seq_to_heads(x, P, transport) for x in (q, k, v, out, dout))
    lh = _seq_to_heads(lse.unsqueeze(-1), P, transport)[..., 0].contiguous()
    dq, dk, dv = blocks.full_backward(qh, kh, vh, oh, lh, gh, causal, scale)
    return tuple(_heads_to_seq(x, P, transport) for x in (dq, dk, dv))


def pass_q_decode(q, k_shard, v_shard, scale=None, src=0, group=None, transport=None,
                  blocks=None):
    """Decode attention of one query token per sequence over a KV cache split
    by token range across the ranks of `group`.

    q        : [B, Hq, 1, d_qk]; rank `src`'s copy is sent to every rank
               (``src=None``: every rank already holds the same q).
    k_shard,
    v_shard  : [B, Hkv, S_r, d] -- this rank's tokens of the cache.  The
               shards need not be equal; an empty shard (S_r = 0) contributes
               nothing.  Which tokens a rank holds does not matter: decode
               has no mask, and the merge does not depend on the order.
    Returns (O [B, Hq, d_v] in q's dtype, LSE fp32 [B, Hq]), the same on
    every rank.

    One gather moves each rank's O_p and LSE_p together: both are written
    into one fp32 slot of B * Hq * (d_v + 1) values, the slots of all ranks
    are gathered, and the stacked partials are taken out of them for the
    merge."""
    P = dist.get_world_size(group)
    transport = transport or default_transport(group)
    blocks = blocks or KernelBlocks()
    B, Hq, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence")
    if src is not None:
        transport.broadcast(q, src)
    dv = v_shard.shape[-1]
    n_o, n_l = B * Hq * dv, B * Hq
    scale = d ** -0.5 if scale is None else scale
    gathered = torch.empty((P, n_o + n_l), device=q.device, dtype=torch.float32)
    slot = torch.empty((n_o + n_l,), device=q.device, dtype=torch.float32)
    o_p, l_p = slot[:n_o].view(B, Hq, dv), slot[n_o:].view(B, Hq)
    if k_shard.shape[2] > 0:
        blocks.decode_partial(q, k_shard, v_shard, scale, o_p, l_p)
    else:  # no tokens here: the empty partial (weight zero in the merge)
        o_p.zero_()
        l_p.fill_(float("-inf"))
    transport.all_gather(gathered, slot)
    o_parts = gathered[:, :n_o].contiguous().view(P, B, Hq, dv)
    l_parts = gathered[:, n_o:].contiguous().view(P, B, Hq)
    return blocks.decode_merge(o_parts, l_parts, q.dtype)
