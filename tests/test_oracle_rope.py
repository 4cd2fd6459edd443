"""Pins for the oracle's rotary position embedding (oracle/rope.py).

The pages name RoPE without defining it (Striped review, 位置编码处理); the
oracle follows RoFormer's rotation.  Pinned against values fixed by that
definition: the identity at position 0, hand-evaluated rotations for d = 2
and d = 4 (fixing sign, pairing and the frequency exponent), the relation
between the two pairings, the relative-position property that motivates
RoPE, and the equivalence of "rotate at original positions, then stripe" with
"stripe the position ids, then rotate".
"""

import numpy as np
import pytest

from oracle import partition, rope
from oracle.partition import CONTIGUOUS, STRIPED
from oracle.rope import HALF, INTERLEAVED

COS1, SIN1 = 0.5403023058681398, 0.8414709848078965
COS100, SIN100 = 0.8623188722876839, -0.5063656411097588


@pytest.mark.parametrize("pairing", [INTERLEAVED, HALF])
def test_position_zero_is_identity(pairing):
    x = np.random.default_rng(0).standard_normal((3, 5, 16))
    assert np.array_equal(rope.rope(x, np.zeros(5), 10000.0, pairing), x)


def test_d2_rotation_values():
    # d = 2: one pair, theta_0 = 1, so the angle is the position itself.
    x = np.array([[1.0, 0.0], [0.0, 1.0], [0.5, -2.0]])
    got = rope.rope(x, [1, 1, 3], 10000.0, INTERLEAVED)
    want = np.array([[COS1, SIN1], [-SIN1, COS1],
                     [-0.21275623218048828, 2.0505449972308245]])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_d4_frequencies_and_pairings():
    # d = 4, base 10^4: theta = (1, 10^-2); at position 100 pair 1 turns by
    # exactly 1 rad and pair 0 by 100 rad.
    e = np.eye(4)
    got_i = rope.rope(e, [100] * 4, 10000.0, INTERLEAVED)
    # interleaved pairs: (0, 1) and (2, 3)
    np.testing.assert_allclose(got_i[0], [COS100, SIN100, 0, 0], atol=1e-12)
    np.testing.assert_allclose(got_i[1], [-SIN100, COS100, 0, 0], atol=1e-12)
    np.testing.assert_allclose(got_i[2], [0, 0, COS1, SIN1], atol=1e-15)
    np.testing.assert_allclose(got_i[3], [0, 0, -SIN1, COS1], atol=1e-15)
    got_h = rope.rope(e, [100] * 4, 10000.0, HALF)
    # half pairs: (0, 2) and (1, 3)
    np.testing.assert_allclose(got_h[0], [COS100, 0, SIN100, 0], atol=1e-12)
    np.testing.assert_allclose(got_h[1], [0, COS1, 0, SIN1], atol=1e-15)
    np.testing.assert_allclose(got_h[2], [-SIN100, 0, COS100, 0], atol=1e-12)
    np.testing.assert_allclose(got_h[3], [0, -SIN1, 0, COS1], atol=1e-15)


def test_half_is_interleaved_on_regrouped_dimensions():
    d = 16
    x = np.random.default_rng(1).standard_normal((7, d))
    pos = np.arange(7) * 13
    regroup = np.empty(d, dtype=int)          # y[2i] = x[i], y[2i+1] = x[i + d/2]
    regroup[0::2] = np.arange(d // 2)
    regroup[1::2] = np.arange(d // 2) + d // 2
    y = x[:, regroup]
    got = rope.rope(x, pos, 500.0, HALF)
    via = rope.rope(y, pos, 500.0, INTERLEAVED)
    back = np.empty_like(via)
    back[:, regroup] = via
    np.testing.assert_allclose(got, back, rtol=0, atol=1e-14)


@pytest.mark.parametrize("pairing", [INTERLEAVED, HALF])
def test_scores_depend_on_relative_position_only(pairing):
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((2, 1, 32))
    base = rope.rope(q, [40], 10000.0, pairing) @ rope.rope(k, [25], 10000.0, pairing).T
    for shift in (1, 7, 1000, 123456):
        s = (rope.rope(q, [40 + shift], 10000.0, pairing)
             @ rope.rope(k, [25 + shift], 10000.0, pairing).T)
        np.testing.assert_allclose(s, base, rtol=1e-9, atol=1e-9)
    other = rope.rope(q, [41], 10000.0, pairing) @ rope.rope(k, [25], 10000.0, pairing).T
    assert abs((other - base).item()) > 1e-6


@pytest.mark.parametrize("pairing", [INTERLEAVED, HALF])
def test_pair_norms_preserved(pairing):
    x = np.random.default_rng(3).standard_normal((9, 8))
    y = rope.rope(x, np.arange(9) * 1001, 10000.0, pairing)
    a, b = rope.pair_index(8, pairing)
    np.testing.assert_allclose(np.hypot(y[:, a], y[:, b]), np.hypot(x[:, a], x[:, b]), rtol=1e-13)


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
def test_rotate_then_stripe_equals_stripe_positions_then_rotate(layout):
    N, P = 24, 4
    x = np.random.default_rng(4).standard_normal((2, N, 16))
    a = rope.rope_partition(x, P, layout, 10000.0, HALF)
    pos = partition.slot_to_token(N, P, layout)
    b = rope.rope(partition.partition(x, P, layout), pos, 10000.0, HALF)
    np.testing.assert_array_equal(a, b)
