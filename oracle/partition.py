"""Token placement over P virtual shards (oracle; test infrastructure only).

Two placements are defined on the pages:

* contiguous ("Ring"): shard p holds tokens [p*c, (p+1)*c) with c = N/P
  ("ICLR 2024論文解説: Ring Attention", ステップ1: シーケンスの分割;
  Striped review, 分区策略对比: "device 0 holds tokens 0-3, device 1 4-7").
* striped: token t lives on shard t mod P ("Striped Attention" review,
  分区策略对比: "device 0 holds tokens 0, 4, 8, 12; device 1 holds 1, 5, 9, 13").

The pages give only shard membership for the striped case.  Reading taken
(the plainest one consistent with the worked example): inside a shard the
tokens keep ascending order, so token t sits at local index t // P, and the
shards are concatenated in order p = 0..P-1.  The physical ("layout") order
is therefore slot s = shard * c + local.

Zigzag: the pages only name it (the Ring-attention overview page, a
variant that, like striping, rebalances the causal work).  Reading taken
(the standard definition of that layout; not given on the pages): the
sequence is cut into 2P chunks of h = c/2 tokens and shard p holds chunk p
followed by chunk 2P-1-p, so every shard has one early and one late chunk.

``slot_to_token[s]`` is the original token index (its position id) of the
token stored in physical slot s.  Position ids are striped with the same map
(Striped review, 位置编码处理).
"""

import numpy as np

CONTIGUOUS = "contiguous"
STRIPED = "striped"
ZIGZAG = "zigzag"


def shard_len(N, P):
    if P < 1 or N % P != 0:
        raise ValueError(f"N={N} must be a positive multiple of P={P}")
    return N // P


def token_of(shard, local, N, P, layout):
    """Original token index held at (shard, local index)."""
    c = shard_len(N, P)
    if layout == CONTIGUOUS:
        return shard * c + local
    if layout == STRIPED:
        return local * P + shard
    if layout == ZIGZAG:
        if c % 2:
            raise ValueError("zigzag needs an even shard length")
        h = c // 2
        return shard * h + local if local < h else (2 * P - 1 - shard) * h + (local - h)
    raise ValueError(layout)


def slot_to_token(N, P, layout):
    """Position id of every physical slot, as an int64 vector of length N."""
    c = shard_len(N, P)
    out = np.empty(N, dtype=np.int64)
    for shard in range(P):
        for local in range(c):
            out[shard * c + local] = token_of(shard, local, N, P, layout)
    return out


def shard_tokens(N, P, layout):
    """List, per shard, of the original tokens it holds (in local order)."""
    c = shard_len(N, P)
    return [[token_of(p, x, N, P, layout) for x in range(c)] for p in range(P)]


def partition(x, P, layout, axis=-2):
    """Token order -> layout order along ``axis``: out[s] = x[slot_to_token[s]]."""
    N = x.shape[axis]
    perm = slot_to_token(N, P, layout)
    return np.take(x, perm, axis=axis)


def unpartition(x, P, layout, axis=-2):
    """Layout order -> token order along ``axis``: out[slot_to_token[s]] = x[s]."""
    N = x.shape[axis]
    perm = slot_to_token(N, P, layout)
    xm = np.moveaxis(x, axis, 0)
    out = np.empty_like(xm)
    out[perm] = xm
    return np.moveaxis(out, 0, axis)
