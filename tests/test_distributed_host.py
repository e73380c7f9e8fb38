"""CPU tests of the multi-device ring and of the Ulysses all-to-all variant
(ring_context_parallelism_ra_b200/distributed.py) over gloo with world sizes
2 and 3.  The block arithmetic is
supplied by the fp64 oracle (a test-only ``blocks`` object), so these tests
check the ring's own logic: the exchange schedule and its pass-KV bytes, the causal skip of a
contiguous split, the striped positions, the final merge, and the routing of
the travelling gradient accumulators back to their owners, and Ulysses' head
re-shard and its inverse, and pass-Q decode (query sent from one rank,
partials gathered and merged on every rank).  Each rank's
result is compared with the oracle's whole-sequence attention and gradients."""
import datetime
import os
import socket
import sys
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBlocks:
    """Block arithmetic from the oracle, for CPU tensors.  Like the library's
    bindings, the merges take densely stacked partials only."""

    @staticmethod
    def _pos(off, stride, n):
        return off + stride * np.arange(n, dtype=np.int64)

    def partial(self, q, k, v, q_offset, k_offset, stride, causal, scale, o, lse):
        from oracle.attention import attention
        oo, ll = attention(q, k, v, scale, causal,
                           q_positions=self._pos(q_offset, stride, q.shape[2]),
                           k_positions=self._pos(k_offset, stride, k.shape[2]))
        o.copy_(torch.from_numpy(oo))
        lse.copy_(torch.from_numpy(ll))

    def merge(self, o_parts, lse_parts, out_dtype, out=None, lse=None):
        from oracle.merge import lse_merge
        assert o_parts.is_contiguous() and lse_parts.is_contiguous()
        oo, ll = lse_merge(o_parts.double().numpy(), lse_parts.double().numpy())
        o, l_ = torch.from_numpy(oo).to(out_dtype), torch.from_numpy(ll).float()
        if out is not None:
            out.copy_(o)
            o = out
        if lse is not None:
            lse.copy_(l_)
            l_ = lse
        return o, l_

    def delta(self, out, dout):
        from oracle.backward import row_delta
        return torch.from_numpy(row_delta(out, dout))

    def full(self, q, k, v, causal, scale):
        from oracle.attention import attention
        oo, ll = attention(q, k, v, scale, causal)
        return torch.from_numpy(oo).to(q.dtype), torch.from_numpy(ll).float()

    def full_backward(self, q, k, v, out, lse, dout, causal, scale):
        from oracle.backward import attention_backward
        return tuple(torch.from_numpy(x).to(q.dtype)
                     for x in attention_backward(q, k, v, dout, scale, causal))

    def decode_partial(self, q, k, v, scale, o_part, lse_part):
        from oracle.attention import attention
        oo, ll = attention(q, k, v, scale, False)
        o_part.copy_(torch.from_numpy(oo[:, :, 0]))
        lse_part.copy_(torch.from_numpy(ll[:, :, 0]))

    def decode_merge(self, o_parts, lse_parts, out_dtype):
        return self.merge(o_parts, lse_parts, out_dtype)

    def backward(self, q, k, v, dout, lse, delta, q_offset, k_offset, stride, causal, scale,
                 dq_acc, dk_acc, dv_acc):
        from oracle.backward import block_backward_share
        a, b, c = block_backward_share(q, k, v, dout, lse, delta, scale, causal,
                                       self._pos(q_offset, stride, q.shape[2]),
                                       self._pos(k_offset, stride, k.shape[2]))
        dq_acc += torch.from_numpy(a).to(dq_acc.dtype)
        dk_acc += torch.from_numpy(b).to(dk_acc.dtype)
        dv_acc += torch.from_numpy(c).to(dv_acc.dtype)


def _counting(base):
    """Wrap a transport so that it counts the bytes this rank sends in ring
    exchanges."""
    class Counting(type(base)):
        sent = 0

        def exchange(self, send, recv, nxt, prv):
            Counting.sent += sum(t.numel() * t.element_size() for t in send)
            return super().exchange(send, recv, nxt, prv)
    return Counting(base.group)


def _rank_main(rank, world, port, striped, causal, errq):
    import torch.distributed as dist

    from oracle.attention import attention
    from oracle.backward import attention_backward
    from oracle.costs import pass_kv_bytes_per_chip
    from ring_context_parallelism_ra_b200.distributed import (HostTransport,
                                                              ring_attention_backward,
                                                              ring_attention_forward)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, L, d, dv = 1, 4, 2, 8, 6, 5
        n = L * world
        rng = np.random.default_rng(1000 + world)
        q = torch.from_numpy(rng.standard_normal((B, Hq, n, d)))
        k = torch.from_numpy(rng.standard_normal((B, Hkv, n, d)))
        v = torch.from_numpy(rng.standard_normal((B, Hkv, n, dv)))
        g = torch.from_numpy(rng.standard_normal((B, Hq, n, dv)))
        rows = (np.arange(rank, n, world) if striped
                else np.arange(rank * L, (rank + 1) * L))
        part = lambda x: x[:, :, rows].contiguous()  # noqa: E731
        scale = 0.4
        tr, blocks = _counting(HostTransport()), OracleBlocks()
        out, lse = ring_attention_forward(part(q), part(k), part(v), causal, scale, striped,
                                          transport=tr, blocks=blocks)
        # pass-KV traffic of the forward: (cp - 1) / cp * S * c_kv bytes per
        # rank, c_kv = the K and V bytes of one token over batch and heads
        c_kv = B * Hkv * (d + dv) * q.element_size()
        assert type(tr).sent == pass_kv_bytes_per_chip(world, n, c_kv)
        want_o, want_l = attention(q, k, v, scale, causal)
        assert np.abs(out.numpy() - want_o[:, :, rows]).max() <= 1e-6
        assert np.abs(lse.numpy() - want_l[:, :, rows]).max() <= 1e-5
        dq, dk, dvv = ring_attention_backward(part(q), part(k), part(v), out, lse, part(g), causal,
                                              scale, striped, transport=tr, blocks=blocks)
        wq, wk, wv = attention_backward(q, k, v, g, scale, causal)
        for got, w in ((dq, wq), (dk, wk), (dvv, wv)):
            assert np.abs(got.numpy() - w[:, :, rows]).max() <= 1e-5 * max(1.0, np.abs(w).max())
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("striped,causal", [(False, True), (True, True), (False, False)])
def test_ring_over_gloo_matches_whole_sequence(world, striped, causal):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, striped, causal, errq))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def _order_main(rank, world, port, errq, outq):
    """Record, on every rank, the order in which the ring backward issues its
    exchanges and block computations, and how many partials the forward
    keeps alive."""
    import torch.distributed as dist

    from ring_context_parallelism_ra_b200.distributed import (HostTransport,
                                                              ring_attention_backward,
                                                              ring_attention_forward)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        events = []

        class Rec(HostTransport):
            def exchange(self, send, recv, nxt, prv):
                # the travelling accumulators are fp32, K and V fp64 here
                events.append("acc" if send[0].dtype == torch.float32 else "kv")
                return super().exchange(send, recv, nxt, prv)

        class RecBlocks(OracleBlocks):
            def backward(self, *args):
                events.append("block")
                return super().backward(*args)

            def merge(self, o_parts, lse_parts, out_dtype, out=None, lse=None):
                events.append(("merge", o_parts.shape[0]))
                return super().merge(o_parts, lse_parts, out_dtype, out, lse)

        L, d = 4, 3
        rng = np.random.default_rng(7)
        x = lambda h: torch.from_numpy(rng.standard_normal((1, h, L, d)))  # noqa: E731
        q, k, v, g = x(2), x(1), x(1), x(2)
        out, lse = ring_attention_forward(q, k, v, False, 0.5, transport=Rec(), blocks=RecBlocks())
        fwd = list(events)
        events.clear()
        ring_attention_backward(q, k, v, out, lse, g, False, 0.5, transport=Rec(),
                                blocks=RecBlocks())
        outq.put((rank, fwd, list(events)))
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_folds_as_it_goes_and_overlaps_the_accumulator_hop(world):
    ctx = mp.get_context("spawn")
    errq, outq = ctx.Queue(), ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_order_main, args=(r, world, port, errq, outq))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    res = [outq.get(timeout=10) for _ in range(world)]
    for rank, fwd, bwd in res:
        # forward: every block after the first is folded into the running
        # result at once (two partials), never all P at the end
        assert [e for e in fwd if e != "kv"] == [("merge", 2)] * (world - 1), (rank, fwd)
        # backward, per step s: the next K/V leave (s < P - 1), then the
        # accumulator of step s - 1 leaves (s > 0) -- both before this
        # step's block is computed -- and a last hop returns the owner's sums
        want = []
        for s in range(world):
            if s < world - 1:
                want.append("kv")
            if s > 0:
                want.append("acc")
            want.append("block")
        want.append("acc")
        assert bwd == want, (rank, bwd)


def _ulysses_main(rank, world, port, errq):
    import torch.distributed as dist

    from oracle.attention import attention
    from oracle.backward import attention_backward
    from ring_context_parallelism_ra_b200.distributed import (HostTransport, pass_q_decode,
                                                              ring_attention_forward,
                                                              ulysses_attention_backward,
                                                              ulysses_attention_forward)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, L, d, dv = 2, 7, 5, 4
        Hq, Hkv = 2 * world, world
        n = L * world
        rng = np.random.default_rng(2000 + world)
        q = torch.from_numpy(rng.standard_normal((B, Hq, n, d)))
        k = torch.from_numpy(rng.standard_normal((B, Hkv, n, d)))
        v = torch.from_numpy(rng.standard_normal((B, Hkv, n, dv)))
        g = torch.from_numpy(rng.standard_normal((B, Hq, n, dv)))
        rows = np.arange(rank * L, (rank + 1) * L)
        part = lambda x: x[:, :, rows].contiguous()  # noqa: E731
        tr, blocks = HostTransport(), OracleBlocks()
        out, lse = ulysses_attention_forward(part(q), part(k), part(v), True, 0.4,
                                             transport=tr, blocks=blocks)
        want_o, want_l = attention(q, k, v, 0.4, True)
        assert out.shape == (B, Hq, L, dv) and lse.shape == (B, Hq, L)
        assert np.abs(out.numpy() - want_o[:, :, rows]).max() <= 1e-6
        assert np.abs(lse.numpy() - want_l[:, :, rows]).max() <= 1e-5
        grads = ulysses_attention_backward(part(q), part(k), part(v), out, lse, part(g), True, 0.4,
                                           transport=tr, blocks=blocks)
        want = attention_backward(q, k, v, g, 0.4, True)
        for got, w in zip(grads, want):
            assert np.abs(got.numpy() - w[:, :, rows]).max() <= 1e-9
        # argument errors are raised on every rank before any exchange
        odd = torch.zeros((B, world + 1, L, d), dtype=torch.float64)
        with pytest.raises(ValueError, match="divisible"):
            ulysses_attention_forward(odd, odd, odd, True, 0.4, transport=tr, blocks=blocks)
        with pytest.raises(ValueError, match="disagree"):
            ring_attention_forward(part(q), part(k)[:, :, :-1], part(v), True, 0.4, transport=tr,
                                   blocks=blocks)
        with pytest.raises(ValueError, match="one query token"):
            pass_q_decode(part(q), part(k), part(v), 0.4, transport=tr, blocks=blocks)
        # the group is still in step: one more exchange completes
        out2, _ = ulysses_attention_forward(part(q), part(k), part(v), True, 0.4,
                                            transport=tr, blocks=blocks)
        assert torch.equal(out2, out)
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ulysses_over_gloo_matches_whole_sequence(world):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ulysses_main, args=(r, world, port, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def _decode_main(rank, world, port, sizes, errq):
    import torch.distributed as dist

    from oracle.attention import attention
    from ring_context_parallelism_ra_b200.distributed import HostTransport, pass_q_decode
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, d, dv = 2, 4, 2, 6, 5
        n = sum(sizes)
        rng = np.random.default_rng(3000 + world)
        q = torch.from_numpy(rng.standard_normal((B, Hq, 1, d)))
        k = torch.from_numpy(rng.standard_normal((B, Hkv, n, d)))
        v = torch.from_numpy(rng.standard_normal((B, Hkv, n, dv)))
        lo = sum(sizes[:rank])
        shard = slice(lo, lo + sizes[rank])
        # only rank 1 holds the real query; the others must receive it
        mine = q.clone() if rank == 1 else torch.full_like(q, 7.0)
        out, lse = pass_q_decode(mine, k[:, :, shard].contiguous(), v[:, :, shard].contiguous(),
                                 0.3, src=1, transport=HostTransport(), blocks=OracleBlocks())
        want_o, want_l = attention(q, k, v, 0.3, False)
        assert torch.equal(mine, q)
        assert out.shape == (B, Hq, dv) and lse.shape == (B, Hq)
        assert np.abs(out.numpy() - want_o[:, :, 0]).max() <= 1e-6
        assert np.abs(lse.numpy() - want_l[:, :, 0]).max() <= 1e-5
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("sizes", [(9, 14), (5, 0, 11)])
def test_pass_q_decode_over_gloo_matches_whole_cache(sizes):
    world = len(sizes)
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_main, args=(r, world, port, sizes, errq))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def _subgroup_main(rank, world, port, errq):
    import torch.distributed as dist

    from oracle.attention import attention
    from ring_context_parallelism_ra_b200.distributed import (HostTransport, pass_q_decode,
                                                              ring_attention_forward)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # two independent rings, {0, 1} and {2, 3}, each on its own sequence:
        # point-to-point calls need global ranks, the ring uses group ranks
        groups = [dist.new_group([0, 1]), dist.new_group([2, 3])]
        gi = rank // 2
        grp, me = groups[gi], rank % 2
        B, Hq, Hkv, L, d, dv = 1, 2, 1, 6, 4, 3
        n = 2 * L
        rng = np.random.default_rng(4000 + gi)
        q = torch.from_numpy(rng.standard_normal((B, Hq, n, d)))
        k = torch.from_numpy(rng.standard_normal((B, Hkv, n, d)))
        v = torch.from_numpy(rng.standard_normal((B, Hkv, n, dv)))
        rows = np.arange(me * L, (me + 1) * L)
        part = lambda x: x[:, :, rows].contiguous()  # noqa: E731
        out, lse = ring_attention_forward(part(q), part(k), part(v), True, 0.5, group=grp,
                                          transport=HostTransport(grp), blocks=OracleBlocks())
        want_o, want_l = attention(q, k, v, 0.5, True)
        assert np.abs(out.numpy() - want_o[:, :, rows]).max() <= 1e-6
        assert np.abs(lse.numpy() - want_l[:, :, rows]).max() <= 1e-5
        # pass-Q decode inside the group, query sent from group rank 1
        qd = q[:, :, :1].clone() if me == 1 else torch.zeros_like(q[:, :, :1])
        od, ld = pass_q_decode(qd, part(k), part(v), 0.5, src=1, group=grp,
                               transport=HostTransport(grp), blocks=OracleBlocks())
        wo, wl = attention(q[:, :, :1], k, v, 0.5, False)
        assert np.abs(od.numpy() - wo[:, :, 0]).max() <= 1e-6
        assert np.abs(ld.numpy() - wl[:, :, 0]).max() <= 1e-5
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def test_rings_on_process_subgroups():
    world = 4
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_subgroup_main, args=(r, world, port, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def _dead_peer_main(rank, world, port, outq):
    import time

    import torch.distributed as dist

    from ring_context_parallelism_ra_b200.distributed import HostTransport, ring_attention_forward
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(0)          # leaves between steps: nothing of it is in flight
    q = torch.zeros((1, 1, 4, 2), dtype=torch.float64)
    t0 = time.time()
    try:
        ring_attention_forward(q, q, q, True, 1.0, transport=HostTransport(),
                               blocks=OracleBlocks())
        outq.put(("no error", time.time() - t0))
    except Exception as e:  # noqa: BLE001
        outq.put((type(e).__name__, time.time() - t0))
    outq.close()
    outq.join_thread()       # the result must leave before the hard exit below
    os._exit(0)


def test_ring_reports_a_dead_peer_instead_of_hanging():
    ctx = mp.get_context("spawn")
    outq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dead_peer_main, args=(r, 2, port, outq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode is not None for p in procs), "a rank hung"
    kind, seconds = outq.get(timeout=5)
    assert kind != "no error" and seconds < 60, (kind, seconds)


def test_nccl_transport_addresses_global_ranks_of_a_subgroup(monkeypatch):
    # NCCL needs GPUs; a recording stand-in for torch.distributed checks the
    # calls the transport makes: peers and roots are global ranks of the group
    import types

    from ring_context_parallelism_ra_b200 import distributed as D

    calls = []

    def isend(*a, **k):
        raise AssertionError("the transport batches its point-to-point calls")

    def irecv(*a, **k):
        raise AssertionError("the transport batches its point-to-point calls")

    class P2POp:
        def __init__(self, op, t, peer, group):
            self.op, self.peer = ("send" if op is isend else "recv"), peer

    fake = types.SimpleNamespace(
        P2POp=P2POp, isend=isend, irecv=irecv,
        batch_isend_irecv=lambda ops: calls.append(("batch", [(o.op, o.peer) for o in ops])) or [],
        get_global_rank=lambda group, r: {0: 4, 1: 6, 2: 7}[r],   # group ranks -> global 4, 6, 7
        broadcast=lambda t, src, group=None: calls.append(("broadcast", src)),
        all_gather_into_tensor=lambda out, inp, group=None: calls.append(
            ("all_gather", tuple(out.shape), tuple(inp.shape))),
    )
    monkeypatch.setattr(D, "dist", fake)
    tr = D.NcclTransport(group="g")
    tr.exchange([torch.zeros(2), torch.zeros(3)], [torch.zeros(2), torch.zeros(3)],
                nxt=2, prv=1).wait()
    tr.broadcast(torch.zeros(1), src=2)
    tr.all_gather(torch.zeros(3, 5), torch.zeros(5))
    assert [c[0] for c in calls] == ["batch", "broadcast", "all_gather"]
    assert calls[0][1] == [("send", 7), ("send", 7), ("recv", 6), ("recv", 6)]
    assert calls[1] == ("broadcast", 7)
    assert calls[2] == ("all_gather", (3, 5), (5,))
