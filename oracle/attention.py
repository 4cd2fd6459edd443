"""Plain causal attention, the quantity the blockwise method must reproduce.

Test infrastructure only (see the package docstring).

Definition ("Striped Attention: Faster Ring Attention for Causal Transformers"
review, section 三 技术架构 / 核心公式):

    CausalAttn(Q, K, V) = Softmax(Q K^T + C) V,
    C[i, t] = -inf if i < t (query before key) else 0,

with the scores scaled as S = Q K^T / sqrt(d) ("ICLR 2024論文解説: Ring
Attention", ステップ3, legend of S_j; the 実装例 uses scale = d_k ** -0.5).
Reading taken: the scale is a parameter, applied before C is added; the
causal comparison is between ORIGINAL token positions (so a permuted layout
is handled by passing the position ids of the rows), and

    lse[i] = ln sum_t exp(S[i, t] + C[i, t])

(natural log, scale included) is returned beside O, since the partial
results of the method are merged through exactly this per-row normaliser
(1cademy page "Computing Attention Weights in Sequence Parallelism").

The whole score matrix is materialised per (batch, head).  ``attention_rows``
evaluates the same per-row definition for a chosen subset of query rows, for
sequences too long to materialise.
"""

import numpy as np


def _as64(a):
    return np.asarray(a, dtype=np.float64)


def _row_softmax_attention(s, v):
    """Given masked scores s [n, m] (-inf = masked) and v [m, dv]: (O, lse)."""
    mx = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - mx)
    den = np.sum(e, axis=-1, keepdims=True)
    o = (e / den) @ v
    lse = (mx + np.log(den))[..., 0]
    return o, lse


def attention(q, k, v, scale, causal, q_pos=None, k_pos=None):
    """O, lse of Softmax(Q K^T * scale + C) V.

    q: [..., Nq, d], k: [..., Nk, d], v: [..., Nk, dv] (any float dtype; the
    computation is float64).  q_pos / k_pos: original token position of each
    row (default 0..N-1).  Returns O [..., Nq, dv] float64 and lse [..., Nq].
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    nq, nk = q.shape[-2], k.shape[-2]
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * float(scale)
    if causal:
        qp = np.arange(nq) if q_pos is None else np.asarray(q_pos)
        kp = np.arange(nk) if k_pos is None else np.asarray(k_pos)
        blocked = kp[None, :] > qp[:, None]
        s = np.where(blocked, -np.inf, s)
    return _row_softmax_attention(s, v)


def attention_rows(q, k, v, scale, causal, rows):
    """The same definition for query rows ``rows`` of one (batch, head) only.

    q, k, v: [N, d] in token order; rows: integer token indices.  Each row is
    computed against all keys it may attend to (keys 0..row when causal).
    Returns O [len(rows), dv] and lse [len(rows)].
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    rows = np.asarray(rows, dtype=np.int64)
    o = np.empty((rows.size, v.shape[-1]))
    lse = np.empty(rows.size)
    for n, i in enumerate(rows):
        kk = k[: i + 1] if causal else k
        vv = v[: i + 1] if causal else v
        s = (kk @ q[i]) * float(scale)
        oi, li = _row_softmax_attention(s[None, :], vv)
        o[n] = oi[0]
        lse[n] = li[0]
    return o, lse


def local_only_attention(q, k, v, scale, causal, P, shard_of_row, q_pos=None):
    """Per-shard attention that never sees the other shards' keys.

    This is the flawed scheme of the 1cademy page ("Flawed Parallel Attention
    Implementation": each GPU attends only to its own segment, so the softmax
    denominator misses the other nodes' partial sums).  It exists as a
    negative control: for P >= 2 it must NOT equal ``attention``.
    q, k, v: [N, d] in layout order; shard_of_row[s] is the shard of slot s.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    n = q.shape[0]
    pos = np.arange(n) if q_pos is None else np.asarray(q_pos)
    o = np.empty((n, v.shape[-1]))
    lse = np.empty(n)
    shard_of_row = np.asarray(shard_of_row)
    for p in range(P):
        idx = np.nonzero(shard_of_row == p)[0]
        o_p, l_p = attention(q[idx], k[idx], v[idx], scale, causal, pos[idx], pos[idx])
        o[idx] = o_p
        lse[idx] = l_p
    return o, lse
