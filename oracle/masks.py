"""Block masks of the two layouts (oracle; test infrastructure only).

Source: "Striped Attention: Faster Ring Attention for Causal Transformers"
review, GetMask 函数 (procedures GETMASKRINGATTENTION and
GETMASKSTRIPEDATTENTION), and the causal matrix C of 三 技术架构 / 核心公式.

Reading taken (the pages are ambiguous here): (j, k) = (query block, key
block).  The printed rules only agree with C when the MASK is indexed as
MASK[x, y] with x = KEY-local index and y = QUERY-local index:

* ring:    j < k: everything blocked; j = k: blocked where y < x (the query
  precedes the key); j > k: nothing blocked.  The ring procedure prints no
  initialisation; it is read as zero-initialised like the striped one.
* striped: j < k: blocked where y <= x; j >= k: blocked where y < x.

Both procedures below return boolean arrays in that printed orientation
(True = -inf).  ``mask_from_positions`` derives the same blocks from the
original token positions and C, in the conventional [query, key]
orientation; the pins check that one is the transpose of the other.
"""

import numpy as np

from .partition import CONTIGUOUS, STRIPED, ZIGZAG, token_of


def _key_query_grid(c):
    """Index grids in the printed orientation: x (key-local) down the rows,
    y (query-local) along the columns."""
    return np.arange(c)[:, None], np.arange(c)[None, :]


def getmask_ring(j, k, c):
    """Ring (contiguous) block mask, MASK[x (key), y (query)], True = -inf.

    A later key block (j < k) is hidden entirely, the diagonal block (j = k)
    hides a key that comes after the query (y < x), an earlier block hides
    nothing."""
    x, y = _key_query_grid(c)
    return np.broadcast_to((j < k) | ((j == k) & (y < x)), (c, c)).copy()


def getmask_striped(j, k, c):
    """Striped block mask, MASK[x (key), y (query)], True = -inf.

    Every block pair has the same shape of mask, a triangle whose diagonal is
    hidden only when the key shard comes after the query shard: hidden where
    y < x + e, with e = 1 for j < k and e = 0 for j >= k."""
    x, y = _key_query_grid(c)
    e = 1 if j < k else 0
    return y < x + e


def getmask_zigzag(j, k, c, P):
    """The zigzag layout has no printed GetMask; its block mask in the same
    MASK[x (key), y (query)] orientation, from C over the token positions."""
    N = c * P
    qpos = np.array([token_of(j, y, N, P, ZIGZAG) for y in range(c)])
    kpos = np.array([token_of(k, x, N, P, ZIGZAG) for x in range(c)])
    return kpos[:, None] > qpos[None, :]


def getmask(j, k, c, layout, P=None):
    if layout == CONTIGUOUS:
        return getmask_ring(j, k, c)
    if layout == STRIPED:
        return getmask_striped(j, k, c)
    if layout == ZIGZAG:
        return getmask_zigzag(j, k, c, P)
    raise ValueError(layout)


def mask_from_positions(j, k, N, P, layout, causal=True):
    """Blocked[query-local, key-local] for query shard j against key shard k,
    taken from C over original token positions."""
    c = N // P
    qpos = np.array([token_of(j, x, N, P, layout) for x in range(c)])
    kpos = np.array([token_of(k, y, N, P, layout) for y in range(c)])
    if not causal:
        return np.zeros((c, c), dtype=bool)
    return kpos[None, :] > qpos[:, None]
