"""Gradients of causal attention (oracle; test infrastructure only).

The pages measure training speedups (Striped review, 五 核心结果) but give no
backward algorithm.  The oracle is the derivative of the plain definition in
``attention.attention`` (Striped review, 核心公式), written out in float64:

    S  = Q K^T * scale + C          P = softmax_row(S)        O = P V
    dV = P^T dO
    dP = dO V^T
    D  = rowsum(dO o O)             (= rowsum(P o dP))
    dS = P o (dP - D)
    dQ = dS K * scale               dK = dS^T Q * scale

with masked entries of P equal to 0.  ``P`` is recomputed from lse
(P = exp(S - lse)), exactly as the forward defined lse.
"""

import numpy as np

from .attention import attention


def attention_backward(q, k, v, do, scale, causal, q_pos=None, k_pos=None):
    """dQ, dK, dV of sum(O * dO) for O = attention(q, k, v); [N, d] arrays."""
    q, k, v, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, do))
    o, lse = attention(q, k, v, scale, causal, q_pos, k_pos)
    nq, nk = q.shape[0], k.shape[0]
    s = (q @ k.T) * float(scale)
    if causal:
        qp = np.arange(nq) if q_pos is None else np.asarray(q_pos)
        kp = np.arange(nk) if k_pos is None else np.asarray(k_pos)
        s = np.where(kp[None, :] > qp[:, None], -np.inf, s)
    p = np.exp(s - lse[:, None])
    dv = p.T @ do
    dp = do @ v.T
    d_row = np.sum(do * o, axis=1)
    ds = p * (dp - d_row[:, None])
    dq = (ds @ k) * float(scale)
    dk = (ds.T @ q) * float(scale)
    return dq, dk, dv, d_row


def dq_rows(q, k, v, do, scale, causal, rows):
    """dQ of the chosen query rows only, by the same definition (row i needs
    its own scores, lse_i, O_i and D_i = dO_i . O_i; nothing of other rows),
    for sequences too long for the full matrices.  [len(rows), d] float64."""
    q, k, v, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, do))
    out = np.empty((len(rows), k.shape[1]))
    for n, i in enumerate(rows):
        nk = (int(i) + 1) if causal else k.shape[0]
        s = (k[:nk] @ q[i]) * float(scale)
        mx = np.max(s)
        e = np.exp(s - mx)
        p = e / np.sum(e)
        o = p @ v[:nk]
        dp = v[:nk] @ do[i]
        ds = p * (dp - np.dot(do[i], o))
        out[n] = (ds @ k[:nk]) * float(scale)
    return out
