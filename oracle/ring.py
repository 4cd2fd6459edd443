"""The blockwise ring method restated step by step, in float64 (oracle).

Test infrastructure only.  Used on tiny inputs to check the method's own
invariants (its result equals the plain definition in ``attention``), never
as the source of expected GPU values at scale.

Steps, in the order of "ICLR 2024論文解説: Ring Attention":

* ステップ1 -- split Q, K, V into P blocks of c = N/P rows (contiguous), or
  stripe them (Striped review, 分区策略对比; see ``partition``).
* ステップ2 -- device j keeps Q_j; in each of P rounds it holds one K/V block
  and passes it on to device j+1, so in round r it holds block (j - r) mod P
  (the 実装例 sends to rank+1 and receives from rank-1).
* ステップ3 -- fold each round in with online softmax.  The printed
  recurrence is incomplete: it shows O_j = diag(l_{j-1}/l_j) O_{j-1} +
  exp(S_j - m_j)/l_j V_j without defining l_j and without the factor that
  re-bases O_{j-1} from the old max to the new one.  Reading taken
  (consistent with the 実装例, which rescales both the running sum and the
  unnormalised output by exp(row_max - new_max)):

      m_j = max(m_{j-1}, rowmax(S_j))
      l_j = exp(m_{j-1} - m_j) l_{j-1} + rowsum(exp(S_j - m_j))
      O_j = diag(exp(m_{j-1} - m_j) l_{j-1} / l_j) O_{j-1}
            + diag(1 / l_j) exp(S_j - m_j) V_j            (normalised form)

  The 実装例 keeps O unnormalised and divides by l once at the end
  (``normalise_each_round=False``); both forms are offered so that the pins
  show they agree.
* Causal blocks are masked with GetMask(j, block) (Striped review, GetMask 函数);
  a row with every key of a block masked contributes nothing to that round
  (the pages are silent; exp(-inf) = 0 with the running max left unchanged).
"""

import numpy as np

from .masks import getmask
from .partition import shard_len


def ring_attention(q, k, v, P, layout, causal, scale, normalise_each_round=False,
                   round_order=None):
    """Blockwise ring attention over P virtual devices.

    q, k, v: [N, d] in LAYOUT order (already partitioned).  Returns O [N, dv]
    and lse [N] in layout order.  ``round_order``: optional permutation of
    range(P) giving the order in which the rounds are folded in (the merge is
    order-independent; the ring order is the default).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[0]
    c = shard_len(N, P)
    out = np.empty((N, v.shape[1]))
    lse_out = np.empty(N)
    rounds = list(range(P)) if round_order is None else list(round_order)
    for j in range(P):                       # device j, its Q block stays put
        qj = q[j * c:(j + 1) * c]
        m = np.full(c, -np.inf)
        l = np.zeros(c)
        o = np.zeros((c, v.shape[1]))
        for r in rounds:
            kb = (j - r) % P                 # block held by device j in round r
            kj = k[kb * c:(kb + 1) * c]
            vj = v[kb * c:(kb + 1) * c]
            s = (qj @ kj.T) * float(scale)
            if causal:
                blocked = getmask(j, kb, c, layout, P).T   # -> [query, key]
                s = np.where(blocked, -np.inf, s)
            m_new = np.maximum(m, np.max(s, axis=1))
            m_sub = np.where(np.isneginf(m_new), 0.0, m_new)
            p = np.exp(s - m_sub[:, None])
            alpha = np.exp(m - m_sub)
            l_new = alpha * l + np.sum(p, axis=1)
            if normalise_each_round:
                with np.errstate(invalid="ignore", divide="ignore"):
                    keep = np.where(l_new > 0, alpha * l / l_new, 0.0)
                    inv = np.where(l_new > 0, 1.0 / l_new, 0.0)
                o = keep[:, None] * o + inv[:, None] * (p @ vj)
            else:
                o = alpha[:, None] * o + p @ vj
            m, l = m_new, l_new
        if not normalise_each_round:
            o = o / l[:, None]
        out[j * c:(j + 1) * c] = o
        lse_out[j * c:(j + 1) * c] = m + np.log(l)
    return out, lse_out


def block_attention(qj, kb_k, kb_v, j, kb, P, layout, causal, scale):
    """One round of one device: query block j against key/value block kb,
    normalised over that block alone.

    Returns (O_r [c, dv], lse_r [c]); a row that sees no key of the block
    (GetMask hides all of them) gets O_r = 0, lse_r = -inf, so that it
    contributes nothing when merged (1cademy page, per-node partial sums;
    the pages are silent on empty rows).
    """
    qj = np.asarray(qj, dtype=np.float64)
    kk = np.asarray(kb_k, dtype=np.float64)
    vv = np.asarray(kb_v, dtype=np.float64)
    c = qj.shape[0]
    s = (qj @ kk.T) * float(scale)
    if causal:
        s = np.where(getmask(j, kb, c, layout, P).T, -np.inf, s)
    mx = np.max(s, axis=1)
    empty = np.isneginf(mx)
    e = np.exp(s - np.where(empty, 0.0, mx)[:, None])
    den = np.sum(e, axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = np.where(empty[:, None], 0.0, (e @ vv) / den[:, None])
        lse = np.where(empty, -np.inf, mx + np.log(den))
    return o, lse


def ring_by_merge(q, k, v, P, layout, causal, scale):
    """The ring with per-round partial results merged through their
    normalisers (1cademy page, "Computing Attention Weights in Sequence
    Parallelism") instead of an online-softmax state: device j merges
    block_attention(j, (j - r) mod P) for r = 0..P-1.  Layout order in and
    out, as ``ring_attention``."""
    from .merge import lse_merge

    q = np.asarray(q, dtype=np.float64)
    N = q.shape[0]
    c = shard_len(N, P)
    out = np.empty((N, np.asarray(v).shape[1]))
    lse_out = np.empty(N)
    for j in range(P):
        o_acc, l_acc = None, None
        for r in range(P):
            kb = (j - r) % P
            o_r, l_r = block_attention(q[j * c:(j + 1) * c], k[kb * c:(kb + 1) * c],
                                       v[kb * c:(kb + 1) * c], j, kb, P, layout, causal, scale)
            if o_acc is None:
                o_acc, l_acc = o_r, l_r
            else:
                o_acc, l_acc = lse_merge(o_acc, l_acc, o_r, l_r)
        out[j * c:(j + 1) * c] = o_acc
        lse_out[j * c:(j + 1) * c] = l_acc
    return out, lse_out
