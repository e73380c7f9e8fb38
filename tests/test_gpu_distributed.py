"""The multi-device ring, the Ulysses variant and pass-Q decode
(distributed.py) with the library's kernels: two ranks
as two processes on one GPU, exchanging K/V and the travelling gradient
accumulators through host memory (gloo, HostTransport).  No kernel waits on
another rank's kernel; only the hosts exchange data.  Each rank's output and
gradients are compared with the fp64 oracle's whole-sequence results."""
import datetime
import math
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

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, errq):
    import torch.distributed as dist

    from oracle.attention import attention
    from oracle.backward import attention_backward
    from ring_context_parallelism_ra_b200 import ra
    from ring_context_parallelism_ra_b200.distributed import (HostTransport,
                                                              ring_attention_backward,
                                                              ring_attention_forward,
                                                              ulysses_attention_backward,
                                                              ulysses_attention_forward)
    from ring_context_parallelism_ra_b200.workloads import make_dout, make_qkv
    from tests.parity_util import check_grad, check_lse, check_out
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        B, Hq, Hkv, L, d = 1, 4, 2, 256, 128
        n = L * world
        q, k, v = make_qkv(B, Hq, Hkv, n, n, d, d, torch.bfloat16, seed=61 + world)
        g = make_dout(B, Hq, n, d, torch.bfloat16, seed=61 + world)
        striped = mode == "striped"
        rows = (np.arange(rank, n, world) if striped
                else np.arange(rank * L, (rank + 1) * L))
        part = lambda x: x[:, :, rows].contiguous().to("cuda")  # noqa: E731
        scale = 1 / math.sqrt(d)
        tr = HostTransport()
        if mode == "ulysses":
            fwd = lambda: ulysses_attention_forward(part(q), part(k), part(v), True, scale,  # noqa: E731
                                                    transport=tr)
            bwd = lambda o, l: ulysses_attention_backward(part(q), part(k), part(v), o, l,  # noqa: E731
                                                          part(g), True, scale, transport=tr)
        else:
            fwd = lambda: ring_attention_forward(part(q), part(k), part(v), True, scale,  # noqa: E731
                                                 striped, transport=tr)
            bwd = lambda o, l: ring_attention_backward(part(q), part(k), part(v), o, l,  # noqa: E731
                                                       part(g), True, scale, striped,
                                                       transport=tr)
        out, lse = fwd()
        want_o, want_l = attention(q, k, v, scale, True)
        check_out(out, want_o[:, :, rows], "bf16")
        check_lse(lse, want_l[:, :, rows])
        dq, dk, dv = bwd(out, lse)
        wq, wk, wv = attention_backward(q, k, v, g, scale, True)
        check_grad(dq, wq[:, :, rows], "bf16", "dQ")
        check_grad(dk, wk[:, :, rows], "bf16", "dK")
        check_grad(dv, wv[:, :, rows], "bf16", "dV")
        assert ra.get_status() == ra.RA_OK
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def _decode_main(rank, world, port, errq):
    import torch.distributed as dist

    from oracle.attention import attention
    from ring_context_parallelism_ra_b200 import ra
    from ring_context_parallelism_ra_b200.distributed import HostTransport, pass_q_decode
    from ring_context_parallelism_ra_b200.workloads import make_qkv
    from tests.parity_util import check_lse, check_out
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        B, Hq, Hkv, d = 2, 16, 2, 128
        sizes = (3000, 5192)                     # ragged shards of an 8192-token cache
        n = sum(sizes)
        q, k, v = make_qkv(B, Hq, Hkv, 1, n, d, d, torch.bfloat16, seed=71)
        lo = sum(sizes[:rank])
        shard = slice(lo, lo + sizes[rank])
        mine = (q if rank == 0 else torch.zeros_like(q)).to("cuda")
        out, lse = pass_q_decode(mine, k[:, :, shard].contiguous().to("cuda"),
                                 v[:, :, shard].contiguous().to("cuda"), d ** -0.5, src=0,
                                 transport=HostTransport())
        want_o, want_l = attention(q, k, v, d ** -0.5, False)
        check_out(out, want_o[:, :, 0], "bf16")
        check_lse(lse, want_l[:, :, 0])
        assert ra.get_status() == ra.RA_OK
    except Exception:
        errq.put((rank, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def test_two_rank_pass_q_decode_on_one_gpu_matches_oracle():
    assert torch.cuda.is_available()
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_main, args=(r, 2, port, errq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


@pytest.mark.parametrize("mode", ["contiguous", "striped", "ulysses"])
def test_two_rank_ring_on_one_gpu_matches_oracle(mode):
    assert torch.cuda.is_available()
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, mode, errq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
