"""The ring across processes: one rank per device, K/V blocks passed around.

"ICLR 2024論文解説: Ring Attention", ステップ2 and its 実装例: device j keeps
its query block Q_j; in each of P rounds it computes with the key/value
block it holds and passes that block to device j+1 while receiving the next
one from device j-1, so that in round r it holds block (j - r) mod P.  The
rounds are combined through their softmax normalisers (1cademy page
"Computing Attention Weights in Sequence Parallelism").  With the striped
layout (Striped review) rank j holds the tokens j, j+P, j+2P, ... and every
round's GetMask keeps the work balanced.

On each rank: ``ra_attn_fwd_block`` computes the round's partial result on
the device (in float32, so that O is rounded to bf16 only once, at the end),
``ra_lse_merge_acc`` folds it into a float32 accumulator, and
the K/V exchange for the next round is posted before the round's compute so
that the transfer overlaps it (``torch.distributed`` point-to-point
operations; NCCL over NVLink on GPUs).  Each rank sends one K and one V block
per round: 2 * B * H * c * d * 2 bytes.

The block and merge steps are parameters so that the exchange logic can be
exercised on host tensors (gloo) with any implementation of those two steps;
by default they are this library's kernels.  A gloo group moves host tensors
only: with device tensors on such a group the blocks are staged through host
buffers (copied out before they are sent, copied in on the current stream
after they arrive), which keeps the device work in stream order.
"""

import torch
import torch.distributed as dist


def _kernels():
    from . import ops

    def block(q, k, v, j, kb, P, layout, causal, scale):
        # float32 partials: O is rounded to bf16 once, by the last merge
        return ops.attn_fwd_block(q, k, v, j, kb, P, layout, causal, scale, o_f32=True)

    return block, ops.lse_merge_acc


def ring_attn_fwd(q, k, v, layout, causal=True, scale=None, group=None, block_fn=None,
                  merge_fn=None, host_staging=None):
    """This rank's share of the ring: q, k, v are the rank's shard
    [B, H, c, d] in layout order (rank j holds shard j of P = world size).
    Returns (o [B, H, c, d] in q's dtype, lse [B, H, c], float32 or wider) of the
    rank's query rows.

    block_fn(q, k, v, j, kb, P, layout, causal, scale) -> (o_r, lse_r) and
    merge_fn(o_acc, lse_acc, o_r, lse_r, first=..., final_out=...) default to
    the library's ``attn_fwd_block`` and ``lse_merge_acc``.  host_staging
    (default: device tensors on a gloo group) sends and receives the K/V
    blocks through host copies.
    """
    if block_fn is None or merge_fn is None:
        kb_fn, mg_fn = _kernels()
        block_fn = block_fn or kb_fn
        merge_fn = merge_fn or mg_fn
    P = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (rank + 1) % P) if group is not None else (rank + 1) % P
    prv = dist.get_global_rank(group, (rank - 1) % P) if group is not None else (rank - 1) % P
    B, H, c, d = q.shape
    if scale is None:
        scale = d ** -0.5
    # float32 accumulator for 16-bit inputs (the kernels' case); wider
    # inputs keep their own precision
    acc = torch.float32 if q.element_size() <= 4 else q.dtype
    o_acc = torch.empty(q.shape, dtype=acc, device=q.device)
    lse_acc = torch.empty((B, H, c), dtype=acc, device=q.device)
    o = torch.empty_like(q)
    if host_staging is None:
        host_staging = q.is_cuda and dist.get_backend(group) == "gloo"
    # Two spare K/V pairs: the block being sent is never the one being
    # received into, and the caller's k, v are never written.
    spare = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    if host_staging:
        # host images of the block being sent and of the one being received
        h_send = [torch.empty(k.shape, dtype=k.dtype) for _ in range(2)]
        h_recv = [torch.empty(k.shape, dtype=k.dtype) for _ in range(2)]
    cur_k, cur_v = k, v
    for r in range(P):
        kb = (rank - r) % P
        reqs = []
        if r < P - 1:
            rk, rv = spare[r % 2]
            if host_staging:
                # the host copies complete before the sends are posted
                h_send[0].copy_(cur_k)
                h_send[1].copy_(cur_v)
                send_k, send_v, recv_k, recv_v = h_send[0], h_send[1], h_recv[0], h_recv[1]
            else:
                send_k, send_v, recv_k, recv_v = cur_k, cur_v, rk, rv
            reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, send_k, nxt, group),
                dist.P2POp(dist.isend, send_v, nxt, group),
                dist.P2POp(dist.irecv, recv_k, prv, group),
                dist.P2POp(dist.irecv, recv_v, prv, group),
            ])
        o_r, lse_r = block_fn(q, cur_k, cur_v, rank, kb, P, layout, causal, scale)
        merge_fn(o_acc, lse_acc, o_r, lse_r, first=(r == 0),
                 final_out=o if r == P - 1 else None)
        for req in reqs:
            req.wait()
        if r < P - 1:
            if host_staging:
                # ordered on the current stream after this round's kernels;
                # synchronous, so the host buffers are free for the next round
                rk.copy_(h_recv[0])
                rv.copy_(h_recv[1])
            cur_k, cur_v = spare[r % 2]
    return o, lse_acc
