"""Planted mistakes: each pin must catch a plausible error in the oracle.

Every test below swaps one oracle function for a copy with a single planted
mistake (a dropped term, a wrong sign or index, a transposed operand) and
checks that at least one pin of test_oracle_*.py then fails.  The mistakes
are planted in the oracle, on the CPU only.
"""

import numpy as np
import pytest

import tests.test_oracle_attention as TA
import tests.test_oracle_partition_masks_work as TP
from oracle import attention as att
from oracle import masks, merge, partition, ring, work
from oracle.partition import CONTIGUOUS, STRIPED


def _attention_mutant(kind):
    def f(q, k, v, scale, causal, q_pos=None, k_pos=None):
        q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
        nq, nk = q.shape[-2], k.shape[-2]
        if kind == "transposed":
            s = np.matmul(k, np.swapaxes(q, -1, -2)) * scale
        elif kind == "no_scale":
            s = np.matmul(q, np.swapaxes(k, -1, -2))
        else:
            s = np.matmul(q, np.swapaxes(k, -1, -2)) * scale
        if causal:
            qp = np.arange(nq) if q_pos is None else np.asarray(q_pos)
            kp = np.arange(nk) if k_pos is None else np.asarray(k_pos)
            if kind == "mask_includes_diagonal":
                blocked = kp[None, :] >= qp[:, None]
                blocked[:, 0] = False            # keep row 0 finite
            elif kind == "mask_flipped":
                blocked = kp[None, :] < qp[:, None]
            else:
                blocked = kp[None, :] > qp[:, None]
            s = np.where(blocked, -np.inf, s)
        mx = np.max(s, axis=-1, keepdims=True)
        e = np.exp(s - mx)
        den = np.sum(e, axis=-1, keepdims=True)
        if kind == "no_normalise":
            den = np.ones_like(den)
        o = (e / den) @ v
        lse = (mx + np.log(den))[..., 0]
        return o, lse
    return f


@pytest.mark.parametrize("kind", ["transposed", "no_scale", "mask_includes_diagonal",
                                  "mask_flipped", "no_normalise"])
def test_attention_mutants_fail_brute_force_pin(monkeypatch, kind):
    monkeypatch.setattr(att, "attention", _attention_mutant(kind))
    with pytest.raises(AssertionError):
        for causal in (True, False):
            TA.test_definition_equals_pure_python_brute_force(causal, 7, 4, 5, 0.5)
            TA.test_definition_equals_pure_python_brute_force(causal, 12, 6, 3, 1.3)


def _ring_mutant(kind):
    def f(q, k, v, P, layout, causal, scale, normalise_each_round=False, round_order=None):
        N = q.shape[0]
        c = N // P
        out = np.empty((N, v.shape[1]))
        lse_out = np.empty(N)
        for j in range(P):
            qj = q[j * c:(j + 1) * c]
            m = np.full(c, -np.inf)
            l = np.zeros(c)
            o = np.zeros((c, v.shape[1]))
            for r in range(P):
                kb = (j - r) % P
                kj, vj = k[kb * c:(kb + 1) * c], v[kb * c:(kb + 1) * c]
                s = (qj @ kj.T) * scale
                if causal:
                    blocked = masks.getmask(j, kb, c, layout)
                    if kind != "mask_not_transposed":
                        blocked = blocked.T
                    s = np.where(blocked, -np.inf, s)
                m_new = np.maximum(m, np.max(s, axis=1))
                m_sub = np.where(np.isneginf(m_new), 0.0, m_new)
                p = np.exp(s - m_sub[:, None])
                alpha = np.exp(m - m_sub)
                if kind == "no_rescale":
                    alpha = np.where(np.isneginf(m), 0.0, 1.0)
                if kind == "rescale_sum_only":
                    o = o + p @ vj
                else:
                    o = alpha[:, None] * o + p @ vj
                l = alpha * l + np.sum(p, axis=1)
                m = m_new
            out[j * c:(j + 1) * c] = o / l[:, None]
            lse_out[j * c:(j + 1) * c] = m + np.log(l)
        return out, lse_out
    return f


@pytest.mark.parametrize("kind", ["mask_not_transposed", "no_rescale", "rescale_sum_only"])
def test_ring_mutants_fail_exactness_pin(monkeypatch, kind):
    monkeypatch.setattr(ring, "ring_attention", _ring_mutant(kind))
    with pytest.raises(AssertionError):
        for layout in (CONTIGUOUS, STRIPED):
            TA.test_blockwise_ring_equals_full_softmax(layout, True, 24, 4, False)


def test_partition_mutant_fails_golden(monkeypatch, golden_dir):
    def swapped(shard, local, N, P, layout):
        c = N // P
        return shard * c + local if layout == STRIPED else local * P + shard
    monkeypatch.setattr(partition, "token_of", swapped)
    with pytest.raises(AssertionError):
        TP.test_worked_stripe_example(golden_dir)


def test_getmask_mutant_fails_position_pin(monkeypatch):
    def wrong(j, k, c):
        mask = np.zeros((c, c), dtype=bool)
        for x in range(c):
            for y in range(c):
                if (j < k and y < x) or (j >= k and y <= x):   # strictness swapped
                    mask[x, y] = True
        return mask
    monkeypatch.setattr(masks, "getmask_striped", wrong)
    with pytest.raises(AssertionError):
        TP.test_getmask_equals_causal_C_over_positions(STRIPED, 3, 4)


def test_work_mutant_fails_brute_force_pin(monkeypatch):
    monkeypatch.setattr(work, "work_striped_printed",
                        lambda i, j, c: c * (c - 1) // 2 if i >= j else c * (c + 1) // 2)
    with pytest.raises(AssertionError):
        TP.test_work_counts_brute_force_equal_closed_forms(STRIPED, 3, 4)


def test_merge_mutant_fails_split_pin(monkeypatch):
    def wrong(o_a, lse_a, o_b, lse_b):
        lse = np.logaddexp(lse_a, lse_b)
        return (np.exp(lse_a)[..., None] * o_a + np.exp(lse_b)[..., None] * o_b), lse
    monkeypatch.setattr(merge, "lse_merge", wrong)
    with pytest.raises(AssertionError):
        TA.test_lse_merge_of_key_halves_equals_full(7)


def _backward_mutant(kind):
    def f(q, k, v, do, scale, causal, q_pos=None, k_pos=None):
        q, k, v, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, do))
        o, lse = att.attention(q, k, v, scale, causal)
        n = q.shape[0]
        s = (q @ k.T) * scale
        if causal:
            s = np.where(np.triu(np.ones((n, n), bool), 1), -np.inf, s)
        p = np.exp(s - lse[:, None])
        dv = p.T @ do
        dp = do @ v.T
        d_row = np.sum(do * o, axis=1)
        ds = p * dp if kind == "no_D" else p * (dp - d_row[:, None])
        dq = (ds @ k) * scale
        dk = (ds @ q) * scale if kind == "dk_untransposed" else (ds.T @ q) * scale
        if kind == "dv_no_transpose":
            dv = p @ do
        return dq, dk, dv, d_row
    return f


@pytest.mark.parametrize("kind", ["no_D", "dk_untransposed", "dv_no_transpose"])
def test_backward_mutants_fail_autograd_pin(monkeypatch, kind):
    import tests.test_oracle_backward as TB
    from oracle import backward as OB
    monkeypatch.setattr(OB, "attention_backward", _backward_mutant(kind))
    with pytest.raises(AssertionError):
        TB.test_backward_equals_torch_autograd(True, 9, 8)


def _rope_mutant(kind):
    from oracle import rope as R

    def f(x, pos, base=10000.0, pairing=R.INTERLEAVED):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        i = np.arange(d // 2, dtype=np.float64)
        expo = -i / d if kind == "freq_exponent" else -2.0 * i / d
        ang = np.asarray(pos, dtype=np.float64)[:, None] * np.power(float(base), expo)[None, :]
        cos, sin = np.cos(ang), np.sin(ang)
        use = R.HALF if (kind == "pairing_swapped" and pairing == R.INTERLEAVED) else pairing
        a, b = R.pair_index(d, use)
        u, w = x[..., a], x[..., b]
        out = np.empty_like(x)
        if kind == "sign":
            out[..., a] = u * cos + w * sin
            out[..., b] = -u * sin + w * cos
        else:
            out[..., a] = u * cos - w * sin
            out[..., b] = u * sin + w * cos
        return out
    return f


@pytest.mark.parametrize("kind", ["sign", "freq_exponent", "pairing_swapped"])
def test_rope_mutants_fail_closed_form_pins(monkeypatch, kind):
    import tests.test_oracle_rope as TR
    from oracle import rope as R
    monkeypatch.setattr(R, "rope", _rope_mutant(kind))
    with pytest.raises(AssertionError):
        TR.test_d2_rotation_values()
        TR.test_d4_frequencies_and_pairings()


def test_zigzag_mutant_fails_example_and_balance(monkeypatch):
    """Planted: shard p holds chunk p and chunk 2P-2-p (an off-by-one mirror)."""
    import tests.test_oracle_partition_masks_work as TP2
    orig = partition.token_of

    def wrong(shard, local, N, P, layout):
        if layout != partition.ZIGZAG:
            return orig(shard, local, N, P, layout)
        h = N // P // 2
        return shard * h + local if local < h else ((2 * P - 2 - shard) % (2 * P)) * h + local - h
    monkeypatch.setattr(partition, "token_of", wrong)
    with pytest.raises(AssertionError):
        TP2.test_zigzag_example_N16_P4()


@pytest.mark.parametrize("kind", ["diagonal_inclusive", "order_swapped"])
def test_ring_getmask_mutants_fail_position_pin(monkeypatch, kind):
    def wrong(j, k, c):
        mask = np.zeros((c, c), dtype=bool)
        hidden = (j > k) if kind == "order_swapped" else (j < k)
        if hidden:
            mask[:, :] = True
        elif j == k:
            for x in range(c):
                for y in range(c):
                    if (y <= x) if kind == "diagonal_inclusive" else (y < x):
                        mask[x, y] = True
        return mask
    monkeypatch.setattr(masks, "getmask_ring", wrong)
    with pytest.raises(AssertionError):
        TP.test_getmask_equals_causal_C_over_positions(CONTIGUOUS, 3, 4)


def test_zigzag_getmask_mutant_fails_orientation_pin(monkeypatch):
    """Planted: the mask blocks a key at the query's own position too."""
    def wrong(j, k, c, P):
        N = c * P
        qpos = np.array([partition.token_of(j, y, N, P, partition.ZIGZAG) for y in range(c)])
        kpos = np.array([partition.token_of(k, x, N, P, partition.ZIGZAG) for x in range(c)])
        return kpos[:, None] >= qpos[None, :]
    monkeypatch.setattr(masks, "getmask_zigzag", wrong)
    with pytest.raises(AssertionError):
        TP.test_zigzag_mask_orientation_matches_positions()


def test_key_block_mutant_fails_ring_pass_pin(monkeypatch):
    """Planted: the ring turning the other way (block (j + r) mod P)."""
    monkeypatch.setattr(work, "key_block", lambda j, r, P: (j + r) % P)
    with pytest.raises(AssertionError):
        TP.test_key_block_follows_the_ring_pass(3)


def _block_attention_mutant(kind):
    orig = ring.block_attention

    def f(qj, kb_k, kb_v, j, kb, P, layout, causal, scale):
        if kind == "pair_swapped":
            return orig(qj, kb_k, kb_v, kb, j, P, layout, causal, scale)
        o, lse = orig(qj, kb_k, kb_v, j, kb, P, layout, causal, scale)
        if kind == "empty_lse_zero":
            lse = np.where(np.isneginf(lse), 0.0, lse)
        return o, lse
    return f


@pytest.mark.parametrize("kind", ["pair_swapped", "empty_lse_zero"])
def test_block_attention_mutants_fail_definition_pin(monkeypatch, kind):
    import tests.test_oracle_attention as TA2
    monkeypatch.setattr(ring, "block_attention", _block_attention_mutant(kind))
    with pytest.raises(AssertionError):
        TA2.test_block_attention_empty_rows_and_positions()


def test_ring_by_merge_mutant_fails_exactness_pin(monkeypatch):
    """Planted: the last round's partial is never merged."""
    from oracle.merge import lse_merge
    from oracle.partition import shard_len

    def wrong(q, k, v, P, layout, causal, scale):
        q = np.asarray(q, dtype=np.float64)
        N = q.shape[0]
        c = shard_len(N, P)
        out, lse_out = np.empty((N, np.asarray(v).shape[1])), np.empty(N)
        for j in range(P):
            o_acc = l_acc = None
            for r in range(max(P - 1, 1)):
                kb = (j - r) % P
                o_r, l_r = ring.block_attention(q[j * c:(j + 1) * c], k[kb * c:(kb + 1) * c],
                                                v[kb * c:(kb + 1) * c], j, kb, P, layout,
                                                causal, scale)
                o_acc, l_acc = (o_r, l_r) if o_acc is None else lse_merge(o_acc, l_acc, o_r, l_r)
            out[j * c:(j + 1) * c], lse_out[j * c:(j + 1) * c] = o_acc, l_acc
        return out, lse_out
    monkeypatch.setattr(ring, "ring_by_merge", wrong)
    with pytest.raises(AssertionError):
        TA.test_ring_by_merging_round_partials_equals_full_softmax(STRIPED, True, 24, 4)


def test_dq_rows_mutant_fails_full_backward_pin(monkeypatch):
    """Planted: dQ rows without the softmax scale factor."""
    from oracle import backward as OB
    orig = OB.dq_rows
    monkeypatch.setattr(OB, "dq_rows",
                        lambda q, k, v, do, scale, causal, rows:
                        orig(q, k, v, do, scale, causal, rows) / scale)
    import tests.test_oracle_backward as TB
    with pytest.raises(AssertionError):
        TB.test_dq_rows_equal_full_backward(True)


def test_tile_census_mutant_fails_brute_force_pin(monkeypatch):
    """Planted: the diagonal tiles counted as full instead of partial."""
    orig = work.tile_census_closed_form

    def wrong(j, r, c, P, layout, causal, b):
        skip, full, part = orig(j, r, c, P, layout, causal, b)
        return skip, full + part, 0
    monkeypatch.setattr(work, "tile_census_closed_form", wrong)
    with pytest.raises(AssertionError):
        TP.test_tile_census_brute_force_equals_closed_form(STRIPED, True, 8, 4, 2)


def test_zigzag_work_mutant_fails_brute_force_pin(monkeypatch):
    """Planted: the second chunk's own triangle dropped from the total."""
    monkeypatch.setattr(work, "work_zigzag_device_total",
                        lambda c, P: (c // 2) ** 2 * (2 * P - 1))
    with pytest.raises(AssertionError):
        TP.test_zigzag_work_is_equal_on_every_device(16, 4)


def test_attention_rows_mutant_fails_full_pin(monkeypatch):
    """Planted: a causal row that does not see its own key."""
    orig = att.attention_rows

    def wrong(q, k, v, scale, causal, rows):
        if not causal:
            return orig(q, k, v, scale, causal, rows)
        o = np.empty((len(rows), np.asarray(v).shape[-1]))
        lse = np.empty(len(rows))
        for n, i in enumerate(rows):
            hi = max(int(i), 1)                  # keys 0..i-1 (row 0 keeps key 0)
            o[n], lse[n] = (a[0] for a in att.attention(np.asarray(q)[i:i + 1],
                                                          np.asarray(k)[:hi],
                                                          np.asarray(v)[:hi], scale, False))
        return o, lse
    monkeypatch.setattr(att, "attention_rows", wrong)
    with pytest.raises(AssertionError):
        TA.test_attention_rows_equals_full(True)


def test_negative_control_mutant_fails(monkeypatch):
    """Planted: a 'local-only' scheme that in fact sees every key (so the
    negative control would no longer show the flaw)."""
    monkeypatch.setattr(att, "local_only_attention",
                        lambda q, k, v, scale, causal, P, shard_of_row, q_pos=None:
                        att.attention(q, k, v, scale, causal))
    with pytest.raises(AssertionError):
        TA.test_negative_control_local_only_is_wrong(True)


def test_rope_partition_mutant_fails_position_pin(monkeypatch):
    """Planted: the rotation applied at the slot index after striping, i.e.
    position ids not permuted with the tokens (what the Striped review's
    位置编码处理 warns against)."""
    import tests.test_oracle_rope as TR
    from oracle import rope as R

    def wrong(x, P, layout, base=10000.0, pairing=R.INTERLEAVED):
        xp = partition.partition(x, P, layout)
        return R.rope(xp, np.arange(x.shape[-2]), base, pairing)
    monkeypatch.setattr(R, "rope_partition", wrong)
    with pytest.raises(AssertionError):
        TR.test_rotate_then_stripe_equals_stripe_positions_then_rotate(STRIPED)
