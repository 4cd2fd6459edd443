"""Pins for the backward oracle: torch autograd in float64 (library routine)
and central finite differences on tiny inputs."""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import backward as OB
from oracle import partition as OP


def rand(n, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((n, d)) * s for s in (scale, scale, 1.0, 1.0)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n,d", [(1, 4), (9, 8), (33, 16)])
def test_backward_equals_torch_autograd(causal, n, d):
    q, k, v, do = rand(n, d, n * d, 2.0)
    scale = d ** -0.5
    dq, dk, dv, _ = OB.attention_backward(q, k, v, do, scale, causal)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq[None, None], tk[None, None], tv[None, None], is_causal=causal, scale=scale)[0, 0]
    (out * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def test_backward_equals_finite_differences():
    q, k, v, do = rand(6, 3, 1, 1.5)
    scale = 0.6
    dq, dk, dv, _ = OB.attention_backward(q, k, v, do, scale, True)

    def loss(q_, k_, v_):
        return float(np.sum(OA.attention(q_, k_, v_, scale, True)[0] * do))

    h = 1e-6
    for arr, grad, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        for i in range(arr.shape[0]):
            for j in range(arr.shape[1]):
                args = [q.copy(), k.copy(), v.copy()]
                args[idx][i, j] += h
                up = loss(*args)
                args[idx][i, j] -= 2 * h
                dn = loss(*args)
                assert abs((up - dn) / (2 * h) - grad[i, j]) < 1e-7


def test_backward_with_positions_is_equivariant():
    """Striped layout: gradients of the permuted problem are the permuted
    gradients (the backward of a striped ring returns them in layout order)."""
    N, P = 24, 4
    q, k, v, do = rand(N, 4, 3)
    perm = OP.slot_to_token(N, P, OP.STRIPED)
    g = OB.attention_backward(q, k, v, do, 0.5, True)
    gp = OB.attention_backward(q[perm], k[perm], v[perm], do[perm], 0.5, True, perm, perm)
    for a, b in zip(g, gp):
        np.testing.assert_allclose(b, a[perm], atol=1e-12)


def test_D_is_rowsum_of_P_times_dP():
    q, k, v, do = rand(10, 5, 4)
    _, _, _, d_row = OB.attention_backward(q, k, v, do, 0.4, True)
    o, lse = OA.attention(q, k, v, 0.4, True)
    s = np.where(np.triu(np.ones((10, 10), bool), 1), -np.inf, q @ k.T * 0.4)
    p = np.exp(s - lse[:, None])
    np.testing.assert_allclose(d_row, np.sum(p * (do @ v.T), axis=1), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_dq_rows_equal_full_backward(causal):
    """The per-row dQ equals the full backward's rows (same definition)."""
    g = np.random.default_rng(8)
    n, d = 40, 8
    q, k, v, do = (g.standard_normal((n, d)) for _ in range(4))
    dq, _, _, _ = OB.attention_backward(q, k, v, do, 0.3, causal)
    rows = [0, 1, 17, 39]
    np.testing.assert_allclose(OB.dq_rows(q, k, v, do, 0.3, causal, rows), dq[rows], atol=1e-12)
