"""The process ring with the library's kernels: 2 and 4 ranks, one GPU.

Each rank is its own process with its own CUDA context on cuda:0 and runs
``ring.ring_attn_fwd`` with the default device steps (``ra_attn_fwd_block``
and ``ra_lse_merge_acc``).  The ranks are joined by a gloo process group, so
the K/V blocks of the ring's exchange (send to rank+1, receive from rank-1:
"ICLR 2024論文解説: Ring Attention", ステップ2) travel through host buffers;
the copies, the round's block kernel and the merge kernel are ordered on each
rank's stream.  The ranks' kernels never wait on one another (each launch is
complete in itself; only the host exchange joins the ranks).  The gathered
O and lse must match the fp64 oracle of the plain definition within the
parity tolerances.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, layout, causal, N, H, up, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from long_context_exact_attn_b200 import ops
        from long_context_exact_attn_b200 import ring
        from long_context_exact_attn_b200 import workloads as W

        torch.cuda.set_device(0)
        w = W.Workload("ring_procs", 1, H, N, 128, world, layout, causal, seed=N + world,
                       qk_scale_up=up)
        q, k, v = (t.cuda() for t in W.make_qkv(w))
        c = N // world
        if layout != W.CONTIGUOUS:
            q, k, v = (ops.partition(t, world, layout) for t in (q, k, v))
        mine = [t[:, :, rank * c:(rank + 1) * c].contiguous() for t in (q, k, v)]
        o, lse = ring.ring_attn_fwd(*mine, layout, causal)
        torch.cuda.synchronize()
        fault = ops.device_fault()
        out.put((rank, o.float().cpu().numpy(), lse.float().cpu().numpy(), fault))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal,up", [
    (2, 1, True, 3.0), (2, 0, True, 1.0), (4, 1, True, 1.0), (4, 0, True, 3.0),
    (4, 1, False, 1.0)])
def test_process_ring_with_library_kernels_matches_oracle(world, layout, causal, up):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_exact_attn_b200 import workloads as W
    from oracle import attention as OA
    from oracle import partition as OP

    N, H = 2048, 2
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, layout, causal, N, H, up, q_))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            rank, o, lse, fault = q_.get(timeout=300)
            res[rank] = (o, lse, fault)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert all(res[r][2] == 0 for r in range(world))
    # rank j holds shard j of the layout: concatenate, then back to token order
    o = np.concatenate([res[r][0] for r in range(world)], axis=2)
    lse = np.concatenate([res[r][1] for r in range(world)], axis=2)
    lay = {W.CONTIGUOUS: OP.CONTIGUOUS, W.STRIPED: OP.STRIPED}[layout]
    inv = np.argsort(OP.slot_to_token(N, world, lay))
    o, lse = o[:, :, inv], lse[:, :, inv]
    w = W.Workload("ring_procs", 1, H, N, 128, world, layout, causal, seed=N + world,
                   qk_scale_up=up)
    q, k, v = W.make_qkv(w)
    for h in range(H):
        o_ref, lse_ref = OA.attention(q[0, h].double().numpy(), k[0, h].double().numpy(),
                                      v[0, h].double().numpy(), w.scale, causal)
        err = np.abs(o[0, h] - o_ref)
        assert err.max() <= O_MAX and err.mean() <= O_MEAN, (h, err.max(), err.mean())
        assert np.abs(lse[0, h] - lse_ref).max() <= LSE_MAX
