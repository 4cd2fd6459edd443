"""Pins for the oracle's attention, ring restatement and lse merge.

The plain definition is pinned against (a) brute force in pure Python on tiny
inputs, (b) a library routine (torch's scaled_dot_product_attention on the
CPU in float64), (c) closed forms (constant V, zero Q, row 0).  The blockwise
restatement is pinned against the definition (the pages' exactness claim).
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import merge, partition, ring
from oracle.partition import CONTIGUOUS, STRIPED


def brute_force(q, k, v, scale, causal):
    """Pure-Python loops over math.exp: O and lse, one row at a time."""
    n, m, dv = len(q), len(k), len(v[0])
    o = [[0.0] * dv for _ in range(n)]
    lse = [0.0] * n
    for i in range(n):
        scores = []
        for t in range(m):
            if causal and t > i:
                continue
            scores.append((t, sum(q[i][a] * k[t][a] for a in range(len(q[i]))) * scale))
        mx = max(s for _, s in scores)
        den = sum(math.exp(s - mx) for _, s in scores)
        for t, s in scores:
            w = math.exp(s - mx) / den
            for a in range(dv):
                o[i][a] += w * v[t][a]
        lse[i] = mx + math.log(den)
    return np.array(o), np.array(lse)


def rand_qkv(n, d, seed, m=None, dv=None):
    rng = np.random.default_rng(seed)
    m = n if m is None else m
    dv = d if dv is None else dv
    return (rng.standard_normal((n, d)), rng.standard_normal((m, d)),
            rng.standard_normal((m, dv)))


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n,d,dv,scale", [(1, 3, 2, 0.7), (7, 4, 5, 0.5), (12, 6, 3, 1.3)])
def test_definition_equals_pure_python_brute_force(causal, n, d, dv, scale):
    q, k, v = rand_qkv(n, d, n * 31 + d, dv=dv)
    o, lse = att.attention(q, k, v, scale, causal)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), scale, causal)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_noncausal_rectangular_equals_brute_force():
    q, k, v = rand_qkv(5, 4, 9, m=9, dv=3)
    o, lse = att.attention(q, k, v, 0.4, False)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), 0.4, False)
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_allclose(lse, lb, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_definition_equals_torch_sdpa_float64(causal):
    q, k, v = rand_qkv(64, 16, 3)
    scale = 16 ** -0.5
    o, lse = att.attention(q, k, v, scale, causal)
    t = [torch.from_numpy(a)[None, None] for a in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=causal, scale=scale)
    np.testing.assert_allclose(o, ref[0, 0].numpy(), atol=1e-12)
    # lse via torch.logsumexp of the masked scores (independent library routine)
    s = torch.from_numpy(q @ k.T * scale)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(64, 64, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_constant_v_gives_constant_o(causal):
    q, k, _ = rand_qkv(33, 8, 5)
    row = np.array([0.25, -1.5, 3.0, 7.0])
    v = np.tile(row, (33, 1))
    o, _ = att.attention(q * 4, k * 4, v, 0.3, causal)
    np.testing.assert_allclose(o, np.tile(row, (33, 1)), rtol=0, atol=1e-14)


def test_causal_row0_equals_v0_and_zero_q_closed_form():
    q, k, v = rand_qkv(20, 8, 6)
    o, lse = att.attention(q, k, v, 0.5, True)
    assert np.array_equal(o[0], v[0])
    assert lse[0] == pytest.approx(float(q[0] @ k[0]) * 0.5, abs=1e-15)
    # Q = 0: every visible score is 0 -> uniform weights over the visible keys.
    o0, l0 = att.attention(np.zeros_like(q), k, v, 0.5, True)
    for i in range(20):
        np.testing.assert_allclose(o0[i], v[: i + 1].mean(axis=0), atol=1e-14)
        assert l0[i] == pytest.approx(math.log(i + 1), abs=1e-14)
    o1, l1 = att.attention(np.zeros_like(q), k, v, 0.5, False)
    np.testing.assert_allclose(o1, np.tile(v.mean(axis=0), (20, 1)), atol=1e-14)
    np.testing.assert_allclose(l1, math.log(20), atol=1e-14)


@pytest.mark.parametrize("causal", [True, False])
def test_attention_rows_equals_full(causal):
    q, k, v = rand_qkv(50, 8, 7)
    o, lse = att.attention(q, k, v, 0.35, causal)
    rows = [0, 1, 17, 49, 23]
    orow, lrow = att.attention_rows(q, k, v, 0.35, causal, rows)
    np.testing.assert_allclose(orow, o[rows], atol=1e-13)
    np.testing.assert_allclose(lrow, lse[rows], atol=1e-13)


def test_position_ids_make_attention_permutation_equivariant():
    q, k, v = rand_qkv(24, 4, 8)
    perm = partition.slot_to_token(24, 4, STRIPED)
    o, lse = att.attention(q, k, v, 0.5, True)
    op, lp = att.attention(q[perm], k[perm], v[perm], 0.5, True, perm, perm)
    np.testing.assert_allclose(op, o[perm], atol=1e-13)
    np.testing.assert_allclose(lp, lse[perm], atol=1e-13)


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,P", [(16, 1), (16, 2), (24, 4), (64, 8), (30, 5)])
@pytest.mark.parametrize("normalise", [False, True])
def test_blockwise_ring_equals_full_softmax(layout, causal, N, P, normalise):
    """The method reaches the plain result exactly (Ring Attention explainer,
    ステップ3: no approximation), in both layouts; striped output
    un-permuted equals the contiguous one (Striped review: permutation
    equivariance)."""
    q, k, v = rand_qkv(N, 8, N + P, dv=6)
    q, k = 3 * q, 3 * k                        # large logits: rescales happen
    scale = 8 ** -0.5
    o_ref, lse_ref = att.attention(q, k, v, scale, causal)
    qp, kp, vp = (partition.partition(a, P, layout, axis=0) for a in (q, k, v))
    o, lse = ring.ring_attention(qp, kp, vp, P, layout, causal, scale,
                                 normalise_each_round=normalise)
    np.testing.assert_allclose(partition.unpartition(o, P, layout, axis=0), o_ref, atol=1e-12)
    np.testing.assert_allclose(partition.unpartition(lse, P, layout, axis=0), lse_ref, atol=1e-12)


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
def test_blockwise_merge_is_order_independent(layout):
    N, P = 32, 4
    q, k, v = rand_qkv(N, 4, 99)
    o_ref, lse_ref = att.attention(q, k, v, 0.5, True)
    rng = np.random.default_rng(1)
    qp, kp, vp = (partition.partition(a, P, layout, axis=0) for a in (q, k, v))
    for _ in range(3):
        order = rng.permutation(P)
        o, lse = ring.ring_attention(qp, kp, vp, P, layout, True, 0.5, round_order=order)
        np.testing.assert_allclose(partition.unpartition(o, P, layout, axis=0), o_ref, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_negative_control_local_only_is_wrong(causal):
    """Attention restricted to each shard's own keys misses the other nodes'
    share of the softmax denominator (1cademy, "Flawed Parallel Attention
    Implementation") and must differ from the definition for P >= 2."""
    N, P = 32, 4
    q, k, v = rand_qkv(N, 4, 5)
    o_ref, _ = att.attention(q, k, v, 0.5, causal)
    shard = np.repeat(np.arange(P), N // P)
    o_loc, _ = att.local_only_attention(q, k, v, 0.5, causal, P, shard)
    assert np.max(np.abs(o_loc - o_ref)) > 1e-2
    # ... while with one shard it is the definition itself.
    o1, _ = att.local_only_attention(q, k, v, 0.5, causal, 1, np.zeros(N, dtype=int))
    np.testing.assert_allclose(o1, o_ref, atol=1e-13)


@pytest.mark.parametrize("split", [1, 7, 16, 31])
def test_lse_merge_of_key_halves_equals_full(split):
    q, k, v = rand_qkv(12, 5, split, m=32)
    q = 2 * q
    o, lse = att.attention(q, k, v, 0.6, False)
    oa, la = att.attention(q, k[:split], v[:split], 0.6, False)
    ob, lb = att.attention(q, k[split:], v[split:], 0.6, False)
    om, lm = merge.lse_merge(oa, la, ob, lb)
    np.testing.assert_allclose(om, o, atol=1e-13)
    np.testing.assert_allclose(lm, lse, atol=1e-13)
    # symmetric
    om2, lm2 = merge.lse_merge(ob, lb, oa, la)
    np.testing.assert_allclose(om2, o, atol=1e-13)


def test_lse_merge_empty_sides():
    o = np.array([[1.0, 2.0], [3.0, 4.0]])
    lse = np.array([0.5, -2.0])
    ninf = np.full(2, -np.inf)
    zero = np.zeros_like(o)
    om, lm = merge.lse_merge(o, lse, zero, ninf)
    np.testing.assert_array_equal(om, o)
    np.testing.assert_array_equal(lm, lse)
    om, lm = merge.lse_merge(zero, ninf, zero, ninf)
    np.testing.assert_array_equal(om, zero)
    assert np.all(np.isneginf(lm))


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,P", [(16, 1), (24, 4), (30, 5), (16, 16)])
def test_ring_by_merging_round_partials_equals_full_softmax(layout, causal, N, P):
    """Per-round partial results merged through their normalisers (1cademy
    page: the denominator is a sum of per-node partial sums) reach the plain
    result, including rounds in which a row sees no key (N = P: one row per
    shard)."""
    q, k, v = rand_qkv(N, 8, 3 * N + P, dv=5)
    q, k = 3 * q, 3 * k
    scale = 8 ** -0.5
    o_ref, lse_ref = att.attention(q, k, v, scale, causal)
    qp, kp, vp = (partition.partition(a, P, layout, axis=0) for a in (q, k, v))
    o, lse = ring.ring_by_merge(qp, kp, vp, P, layout, causal, scale)
    np.testing.assert_allclose(partition.unpartition(o, P, layout, axis=0), o_ref, atol=1e-12)
    np.testing.assert_allclose(partition.unpartition(lse, P, layout, axis=0), lse_ref, atol=1e-12)


def test_block_attention_empty_rows_and_positions():
    """A round's partial equals the plain definition over the block's keys
    with the original positions; rows that see none of them are (0, -inf)."""
    N, P = 20, 4
    c = N // P
    q, k, v = rand_qkv(N, 6, 5)
    for layout in (CONTIGUOUS, STRIPED):
        toks = partition.shard_tokens(N, P, layout)
        qp, kp, vp = (partition.partition(a, P, layout, axis=0) for a in (q, k, v))
        for j in range(P):
            for kb in range(P):
                o, lse = ring.block_attention(qp[j * c:(j + 1) * c], kp[kb * c:(kb + 1) * c],
                                              vp[kb * c:(kb + 1) * c], j, kb, P, layout, True, 0.4)
                for x in range(c):
                    vis = [y for y in range(c) if toks[kb][y] <= toks[j][x]]
                    if not vis:
                        assert lse[x] == -np.inf and np.all(o[x] == 0)
                        continue
                    s = np.array([q[toks[j][x]] @ k[toks[kb][y]] * 0.4 for y in vis])
                    w = np.exp(s - s.max())
                    ref_o = (w / w.sum()) @ np.array([v[toks[kb][y]] for y in vis])
                    np.testing.assert_allclose(o[x], ref_o, atol=1e-12)
                    np.testing.assert_allclose(lse[x], s.max() + np.log(w.sum()), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,P", [(16, 2), (24, 4), (40, 5)])
def test_zigzag_ring_equals_full_softmax(causal, N, P):
    """The ring over the zigzag layout (both folds) reaches the plain
    result, like the two layouts of the pages."""
    from oracle.partition import ZIGZAG
    q, k, v = rand_qkv(N, 8, 7 * N + P, dv=6)
    q, k = 3 * q, 3 * k
    o_ref, lse_ref = att.attention(q, k, v, 0.35, causal)
    qp, kp, vp = (partition.partition(a, P, ZIGZAG, axis=0) for a in (q, k, v))
    for o, lse in (ring.ring_attention(qp, kp, vp, P, ZIGZAG, causal, 0.35),
                   ring.ring_by_merge(qp, kp, vp, P, ZIGZAG, causal, 0.35)):
        np.testing.assert_allclose(partition.unpartition(o, P, ZIGZAG, axis=0), o_ref, atol=1e-12)
        np.testing.assert_allclose(partition.unpartition(lse, P, ZIGZAG, axis=0), lse_ref,
                                   atol=1e-12)
