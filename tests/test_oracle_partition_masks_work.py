"""Pins for the oracle's partition, GetMask and work/tile-count functions.

Everything here is integer work and must hold exactly.
"""

import os

import numpy as np
import pytest

from oracle import masks, partition, work
from oracle.partition import CONTIGUOUS, STRIPED


def _read_golden(path):
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, toks = line.split(":")
            layout, dev = head.split()
            rows[(layout, int(dev))] = [int(t) for t in toks.split()]
    return rows


def test_worked_stripe_example(golden_dir):
    """The printed 16-token / 4-device placements (Striped review, 分区策略对比)."""
    rows = _read_golden(os.path.join(golden_dir, "stripe_example_N16_P4.txt"))
    assert rows
    for (layout, dev), toks in rows.items():
        assert partition.shard_tokens(16, 4, layout)[dev] == toks


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("N,P", [(16, 4), (24, 3), (8, 1), (8, 8), (60, 5)])
def test_partition_is_a_permutation_and_inverts(layout, N, P):
    perm = partition.slot_to_token(N, P, layout)
    assert sorted(perm.tolist()) == list(range(N))
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, N, 3))
    y = partition.partition(x, P, layout, axis=1)
    assert np.array_equal(partition.unpartition(y, P, layout, axis=1), x)
    # The partitioned sequence really is shard after shard.
    c = N // P
    for p in range(P):
        for loc in range(c):
            t = partition.token_of(p, loc, N, P, layout)
            assert np.array_equal(y[:, p * c + loc], x[:, t])


def test_striped_membership_is_mod_P():
    N, P = 40, 8
    for p, toks in enumerate(partition.shard_tokens(N, P, STRIPED)):
        assert all(t % P == p for t in toks)
        assert toks == sorted(toks)


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("c,P", [(1, 3), (2, 2), (3, 4), (5, 3), (4, 1)])
def test_getmask_equals_causal_C_over_positions(layout, c, P):
    """GetMask (printed orientation MASK[key, query]) == C from positions."""
    N = c * P
    for j in range(P):
        for k in range(P):
            printed = masks.getmask(j, k, c, layout)
            derived = masks.mask_from_positions(j, k, N, P, layout)
            assert np.array_equal(printed.T, derived), (j, k)


def test_getmask_literal_query_row_reading_is_anticausal():
    """Reading MASK[x, y] with x = query would block the keys BEFORE each query
    on the ring diagonal: the opposite of C.  This is why the transposed
    reading is taken."""
    c = 4
    literal = masks.getmask_ring(0, 0, c)           # as [query, key]
    derived = masks.mask_from_positions(0, 0, c, 1, CONTIGUOUS)
    assert not np.array_equal(literal, derived)
    assert np.array_equal(literal, derived.T)


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("c,P", [(1, 4), (3, 4), (4, 8), (7, 3), (16, 2)])
def test_work_counts_brute_force_equal_closed_forms(layout, c, P):
    N = c * P
    total = 0
    for j in range(P):
        for r in range(P):
            brute = work.work_brute_force(j, r, N, P, layout)
            assert brute == work.work_exact_closed_form(j, r, c, P, layout)
            total += brute
            kb = work.key_block(j, r, P)
            if layout == STRIPED:
                # the printed striped formula holds in every round
                assert brute == work.work_striped_printed(j, kb, c)
            elif r > 0:
                # the printed ring formula holds off the diagonal block
                assert brute == work.work_ring_printed(j, kb, c)
                assert brute in (0, c * c)
            else:
                assert brute == c * (c + 1) // 2
    assert total == N * (N + 1) // 2
    # non-causal: c^2 everywhere
    for j in range(P):
        for r in range(P):
            assert work.work_brute_force(j, r, N, P, layout, causal=False) == c * c


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("c,P,b", [(8, 4, 2), (12, 3, 4), (16, 2, 16), (6, 5, 3)])
def test_tile_census_brute_force_equals_closed_form(layout, causal, c, P, b):
    N = c * P
    for j in range(P):
        for r in range(P):
            skip, full, part, pairs = work.tile_census_brute_force(j, r, N, P, layout, causal, b, b)
            assert (skip, full, part) == work.tile_census_closed_form(j, r, c, P, layout, causal, b)
            assert pairs == work.work_exact_closed_form(j, r, c, P, layout, causal)


def test_striped_balances_per_round_work():
    """Striped: every device does c(c+1)/2 or c(c-1)/2 in every round; ring:
    per-round maximum over devices is c^2 (the imbalance the method fixes)."""
    c, P = 8, 4
    N = c * P
    for r in range(1, P):
        ring = [work.work_brute_force(j, r, N, P, CONTIGUOUS) for j in range(P)]
        strp = [work.work_brute_force(j, r, N, P, STRIPED) for j in range(P)]
        assert max(ring) == c * c and min(ring) == 0
        assert set(strp) <= {c * (c + 1) // 2, c * (c - 1) // 2}


# ------------------------------------------------------------------ zigzag
# The pages only name the zigzag layout; the oracle's reading (chunk p and
# chunk 2P-1-p of 2P chunks on shard p) is pinned here by a hand-written
# example of that definition, the permutation property, the equal work of
# every device and the ring's exactness.
from oracle.partition import ZIGZAG  # noqa: E402


def test_zigzag_example_N16_P4():
    want = [[0, 1, 14, 15], [2, 3, 12, 13], [4, 5, 10, 11], [6, 7, 8, 9]]
    assert partition.shard_tokens(16, 4, ZIGZAG) == want


@pytest.mark.parametrize("N,P", [(16, 4), (24, 3), (8, 1), (16, 8), (60, 5)])
def test_zigzag_partition_is_a_permutation_and_inverts(N, P):
    perm = partition.slot_to_token(N, P, ZIGZAG)
    assert sorted(perm.tolist()) == list(range(N))
    x = np.arange(N * 3).reshape(N, 3)
    assert np.array_equal(partition.unpartition(partition.partition(x, P, ZIGZAG, axis=0), P,
                                                ZIGZAG, axis=0), x)


@pytest.mark.parametrize("N,P", [(16, 4), (24, 3), (40, 5), (32, 8)])
def test_zigzag_work_is_equal_on_every_device(N, P):
    c = N // P
    totals = [sum(work.work_brute_force(j, r, N, P, ZIGZAG) for r in range(P)) for j in range(P)]
    assert totals == [work.work_zigzag_device_total(c, P)] * P
    assert sum(totals) == N * (N + 1) // 2


def test_zigzag_mask_orientation_matches_positions():
    N, P = 24, 3
    c = N // P
    for j in range(P):
        for k in range(P):
            assert np.array_equal(masks.getmask(j, k, c, ZIGZAG, P).T,
                                  masks.mask_from_positions(j, k, N, P, ZIGZAG))


@pytest.mark.parametrize("P", [1, 2, 3, 4, 7])
def test_key_block_follows_the_ring_pass(P):
    """Ring explainer, ステップ2: every device starts with its own K/V block
    and, each round, hands the block it holds to device j+1 (receiving from
    j-1).  Simulating that hand-over round by round gives the block each
    device holds; key_block(j, r, P) must name the same block."""
    held = list(range(P))                       # round 0: own block
    for r in range(P):
        for j in range(P):
            assert work.key_block(j, r, P) == held[j], (j, r)
        held = [held[(j - 1) % P] for j in range(P)]   # receive from j-1
    assert held == list(range(P))               # after P rounds, back home


def _ring_time(c, P, layout, brute):
    """Sum over rounds of the busiest device's unmasked pairs (each round
    lasts as long as its slowest device: Striped review, 问题定义)."""
    total = 0
    for r in range(P):
        if brute:
            total += max(work.work_brute_force(j, r, c * P, P, layout) for j in range(P))
        else:
            total += max(work.work_exact_closed_form(j, r, c, P, layout) for j in range(P))
    return total


def test_striped_speedup_over_ring_approaches_two():
    """Striped review, 理论最大加速比: as the block size and the device count
    grow, Striped over Ring tends to 2x.  Per-round maxima of the exact
    counts give ring = c(c+1)/2 + (P-1) c^2 and striped = P c(c+1)/2; the
    ratio grows with c and P and stays below 2."""
    for c, P in ((1, 2), (3, 4), (8, 3), (6, 6)):
        ring_t, striped_t = _ring_time(c, P, CONTIGUOUS, True), _ring_time(c, P, STRIPED, True)
        assert ring_t == c * (c + 1) // 2 + (P - 1) * c * c
        assert striped_t == P * c * (c + 1) // 2
    prev = 0.0
    for c, P in ((4, 2), (16, 4), (64, 8), (256, 16), (1024, 64), (4096, 256)):
        s = _ring_time(c, P, CONTIGUOUS, False) / _ring_time(c, P, STRIPED, False)
        assert prev < s < 2.0
        prev = s
    assert prev > 1.99
