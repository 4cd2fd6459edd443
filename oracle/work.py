"""Work per device and round, and tile census (oracle; test infrastructure).

Closed forms from "Striped Attention: Faster Ring Attention for Causal
Transformers" review, 三 技术架构:

* Ring Attention 工作负载:  Work_Ring(j, k) = c^2 if j >= k, 0 if j < k
* Striped Attention 工作负载: Work(i, j) = c(c+1)/2 if i >= j, c(c-1)/2 if i < j

Readings taken:

* The index pair is (query device, key block); the key block held by device
  j in round r is (j - r) mod P (ring direction of the Ring Attention 実装例).
* The ring formula ignores the diagonal block: in round 0 (key block = query
  block) the exact count of unmasked pairs is c(c+1)/2, not c^2.  The
  functions below return exact counts; ``work_ring_printed`` keeps the
  printed form for the off-diagonal rounds.
* Non-causal attention masks nothing: c^2 in every round.

Tile census: a block of c x c pairs is cut into tiles of bm x bn (Striped
review, 实现细节 / 分块与分瓦片: a fully masked tile is skipped).  A tile is
"skip" if every pair in it is masked, "full" if none is, "partial"
otherwise.  The ragged tail (c not a multiple of the tile) is counted with
the tile's out-of-range rows ignored.  Reading for a tile cut by the end of
the key block (y0 + bn > c): its columns past the block hold no key of this
block, so computing the tile needs a per-element mask even when every
in-block pair is visible -- it counts as "partial" unless it is skipped.
"""

import numpy as np

from .masks import mask_from_positions
from .partition import CONTIGUOUS, STRIPED


def key_block(j, r, P):
    return (j - r) % P


def work_ring_printed(j, k, c):
    return c * c if j >= k else 0


def work_striped_printed(i, j, c):
    return c * (c + 1) // 2 if i >= j else c * (c - 1) // 2


def work_exact_closed_form(j, r, c, P, layout, causal=True):
    """Unmasked (query, key) pairs on device j in round r, closed form."""
    if not causal:
        return c * c
    kb = key_block(j, r, P)
    if layout == CONTIGUOUS:
        if kb == j:
            return c * (c + 1) // 2
        return work_ring_printed(j, kb, c)
    if layout == STRIPED:
        return work_striped_printed(j, kb, c)
    raise ValueError(layout)


def work_zigzag_device_total(c, P):
    """Visible pairs of one device over all rounds, zigzag layout (the
    reading of the partition module): chunks a and 2P-1-a of h = c/2 tokens
    give sum over their tokens t of (t + 1) = h^2 (2P - 1) + h (h + 1), the
    same for every device (the balance the layout exists for)."""
    h = c // 2
    return h * h * (2 * P - 1) + h * (h + 1)


def work_brute_force(j, r, N, P, layout, causal=True):
    """Unmasked pairs counted element by element from token positions."""
    kb = key_block(j, r, P)
    blocked = mask_from_positions(j, kb, N, P, layout, causal)
    return int(blocked.size - np.count_nonzero(blocked))


def tile_census_brute_force(j, r, N, P, layout, causal, bm, bn):
    """(skip, full, partial, unmasked_pairs) for device j, round r."""
    c = N // P
    kb = key_block(j, r, P)
    blocked = mask_from_positions(j, kb, N, P, layout, causal)
    skip = full = partial = 0
    for x0 in range(0, c, bm):
        for y0 in range(0, c, bn):
            t = blocked[x0:x0 + bm, y0:y0 + bn]
            n_blocked = np.count_nonzero(t)
            if n_blocked == t.size:
                skip += 1
            elif n_blocked == 0 and y0 + bn <= c:
                full += 1
            else:
                partial += 1
    return skip, full, partial, int(blocked.size - np.count_nonzero(blocked))


def tile_census_closed_form(j, r, c, P, layout, causal, b):
    """(skip, full, partial) with square tiles b x b and c a multiple of b.

    T = c / b tiles per side.  Contiguous: round 0 is the diagonal block
    (T partial on the diagonal, T(T-1)/2 full below, T(T-1)/2 skipped
    above); earlier blocks are all full, later blocks all skipped.  Striped:
    every block has the diagonal tiles partial, the lower triangle full and
    the upper triangle skipped.  Non-causal: all T^2 full.
    """
    if c % b:
        raise ValueError("closed form needs c to be a multiple of the tile")
    T = c // b
    tri = T * (T - 1) // 2
    if not causal:
        return 0, T * T, 0
    kb = key_block(j, r, P)
    if layout == CONTIGUOUS:
        if kb == j:
            return tri, tri, T
        if kb < j:
            return 0, T * T, 0
        return T * T, 0, 0
    if layout == STRIPED:
        return tri, tri, T
    raise ValueError(layout)
