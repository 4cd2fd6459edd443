"""The process ring (long_context_exact_attn_b200/ring.py) on CPU ranks over
gloo: the K/V exchange of the Ring explainer (send to rank+1, receive from
rank-1; block (j - r) mod P in round r) and the merge of round partials.

The two device steps are the oracle's (tests may use it): the round partial
``oracle.ring.block_attention`` and the normaliser merge
``oracle.merge.lse_merge``, here on float64 host tensors.  Every rank checks
that the block it holds in round r is block (j - r) mod P of the global
tensors, and the gathered result must equal the plain definition to 1e-12.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, layout, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from long_context_exact_attn_b200 import ring
        from oracle import merge as OM
        from oracle import partition as OP
        from oracle import ring as OR

        N, d, P = 6 * world, 8, world
        c = N // P
        g = np.random.default_rng(11)
        q, k, v = (g.standard_normal((N, d)) * s for s in (3.0, 3.0, 1.0))
        lay = {0: OP.CONTIGUOUS, 1: OP.STRIPED, 2: OP.ZIGZAG}[layout]
        qp, kp, vp = (OP.partition(a, P, lay, axis=0) for a in (q, k, v))
        shard = lambda a, j: torch.from_numpy(np.ascontiguousarray(a[j * c:(j + 1) * c]))[None, None]
        seen = []

        def block_fn(qt, kt, vt, j, kb, P_, layout_, causal_, scale):
            assert np.array_equal(kt[0, 0].numpy(), kp[kb * c:(kb + 1) * c])
            assert np.array_equal(vt[0, 0].numpy(), vp[kb * c:(kb + 1) * c])
            seen.append(kb)
            o, lse = OR.block_attention(qt[0, 0].numpy(), kt[0, 0].numpy(), vt[0, 0].numpy(), j,
                                        kb, P_, lay, causal_, scale)
            return torch.from_numpy(o)[None, None], torch.from_numpy(lse)[None, None]

        def merge_fn(o_acc, lse_acc, o_r, lse_r, first=False, final_out=None):
            if first:
                o_acc.copy_(o_r)
                lse_acc.copy_(lse_r)
            else:
                o, lse = OM.lse_merge(o_acc.numpy(), lse_acc.numpy(), o_r.numpy(), lse_r.numpy())
                o_acc.copy_(torch.from_numpy(o))
                lse_acc.copy_(torch.from_numpy(lse))
            if final_out is not None:
                final_out.copy_(o_acc)

        o, lse = ring.ring_attn_fwd(shard(qp, rank).double(), shard(kp, rank).double(),
                                    shard(vp, rank).double(), layout, causal, d ** -0.5,
                                    block_fn=block_fn, merge_fn=merge_fn)
        assert seen == [(rank - r) % P for r in range(P)]
        out.put((rank, o[0, 0].numpy().copy(), lse[0, 0].numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal", [
    (2, 1, True), (2, 0, True), (2, 1, False), (4, 1, True), (4, 0, True), (4, 1, False),
    (3, 1, True), (2, 2, True), (4, 2, True)])
def test_process_ring_equals_definition(world, layout, causal):
    from oracle import attention as OA
    from oracle import partition as OP

    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, layout, causal, q_))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (o, l)) for r, o, l in (q_.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    N, d, P = 6 * world, 8, world
    g = np.random.default_rng(11)
    q, k, v = (g.standard_normal((N, d)) * s for s in (3.0, 3.0, 1.0))
    lay = {0: OP.CONTIGUOUS, 1: OP.STRIPED, 2: OP.ZIGZAG}[layout]
    o_ref, lse_ref = OA.attention(q, k, v, d ** -0.5, causal)
    o = np.concatenate([res[r][0] for r in range(P)])
    lse = np.concatenate([res[r][1] for r in range(P)])
    np.testing.assert_allclose(OP.unpartition(o, P, lay, axis=0), o_ref, atol=1e-12)
    np.testing.assert_allclose(OP.unpartition(lse, P, lay, axis=0), lse_ref, atol=1e-12)


def _failing_worker(rank, world, port, dead, out):
    """Rank `dead` joins the process group, then fails before its first
    round (an exception on the host, as a crashed data loader would); the
    others run the ring and must end with an error, not wait for ever."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    try:
        if rank == dead:
            raise RuntimeError("planted host failure")
        from long_context_exact_attn_b200 import ring
        from oracle import merge as OM
        from oracle import ring as OR
        from oracle.partition import STRIPED

        c, d = 4, 8
        x = torch.ones(1, 1, c, d, dtype=torch.float64)

        def block_fn(qt, kt, vt, j, kb, P_, layout_, causal_, scale):
            o, lse = OR.block_attention(qt[0, 0].numpy(), kt[0, 0].numpy(), vt[0, 0].numpy(), j,
                                        kb, P_, STRIPED, causal_, scale)
            return torch.from_numpy(o)[None, None], torch.from_numpy(lse)[None, None]

        def merge_fn(o_acc, lse_acc, o_r, lse_r, first=False, final_out=None):
            if first:
                o_acc.copy_(o_r)
                lse_acc.copy_(lse_r)
            else:
                o, lse = OM.lse_merge(o_acc.numpy(), lse_acc.numpy(), o_r.numpy(), lse_r.numpy())
                o_acc.copy_(torch.from_numpy(o))
                lse_acc.copy_(torch.from_numpy(lse))

        ring.ring_attn_fwd(x, x, x, 1, True, d ** -0.5, block_fn=block_fn, merge_fn=merge_fn)
        out.put((rank, "finished"))
    except Exception as e:                      # reported, then the process ends
        out.put((rank, type(e).__name__))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.parametrize("world,dead", [(3, 1), (4, 2)])
def test_ring_rank_failure_ends_every_rank_with_an_error(world, dead):
    """Failure detection on the host (no GPU): when one rank fails, every
    other rank's ring ends with an exception (a peer closed, or the 10 s
    process-group timeout) instead of hanging, and every process exits."""
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, world, port, dead, q_))
             for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = dict(q_.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
        for p in procs:
            if p.is_alive():                    # only the processes this test started
                p.kill()
                p.join(timeout=10)
    assert res[dead] == "RuntimeError"
    for r in range(world):
        assert res[r] != "finished", (r, res)
    for p in procs:
        assert p.exitcode is not None
