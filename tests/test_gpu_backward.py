"""GPU parity of the backward pass (dQ, dK, dV) against the fp64 oracle.

Tolerance (the sources give none for the backward; derived from the
arithmetic): inputs bf16, P and dS rounded to bf16 before their products
(relative 2^-8 at worst), fp32 accumulation, outputs rounded to bf16.  Each
gradient element is a sum of such products, so its error is bounded by a
few 2^-8 of the sum of the absolute terms, which for these inputs stays
within 2 % of the tensor's largest entry; the mean error is an order of
magnitude smaller.  Checked per tensor: max |g - g_ref| <= 2e-2 * max|g_ref|
and mean |g - g_ref| <= 2e-3 * max|g_ref|.
"""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import backward as OB

pytestmark = pytest.mark.gpu

REL_MAX, REL_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


def run_bwd(q, k, v, do, P, layout, causal):
    dev = [t.cuda() for t in (q, k, v, do)]
    if layout != W.CONTIGUOUS:
        dev = [ops.partition(t, P, layout) for t in dev]
    dq_, dk_, dv_, ddo = dev
    o, lse = ops.attn_fwd(dq_, dk_, dv_, P, layout, causal)
    gq, gk, gv = ops.attn_bwd(dq_, dk_, dv_, o, ddo, lse, P, layout, causal)
    if layout != W.CONTIGUOUS:
        gq, gk, gv = (ops.partition(t, P, layout, inverse=True) for t in (gq, gk, gv))
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    return [t.float().cpu().numpy() for t in (gq, gk, gv)]


def check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        scale = max(np.abs(r).max(), 1e-6)
        err = np.abs(g - r)
        assert np.isfinite(g).all(), f"{what} {name}"
        assert err.max() <= REL_MAX * scale, f"{what} {name}: max {err.max() / scale:.3e}"
        assert err.mean() <= REL_MEAN * scale, f"{what} {name}: mean {err.mean() / scale:.3e}"


CASES = [
    # (B, H, N, d, P, layout, causal, qk_scale_up)
    (1, 1, 256, 64, 4, W.CONTIGUOUS, False, 1.0),
    (1, 2, 1024, 128, 4, W.CONTIGUOUS, True, 1.0),
    (1, 2, 1024, 128, 4, W.STRIPED, True, 1.0),
    (2, 1, 600, 128, 3, W.STRIPED, True, 1.0),        # ragged shards
    (1, 2, 1500, 64, 5, W.STRIPED, True, 3.0),
    (1, 1, 2048, 128, 1, W.CONTIGUOUS, True, 3.0),
    (1, 2, 512, 128, 8, W.STRIPED, False, 1.0),
    (1, 1, 4096, 128, 8, W.STRIPED, True, 3.0),       # 4 key tiles per shard
    (1, 1, 4096, 128, 4, W.CONTIGUOUS, True, 1.0),
    (1, 1, 3000, 64, 3, W.CONTIGUOUS, False, 1.0),    # ragged, non-causal
    (1, 2, 4096, 128, 4, W.ZIGZAG, True, 1.0),         # zigzag: chunks j and 2P-1-j
    (2, 1, 2048, 64, 2, W.ZIGZAG, True, 3.0),
    (1, 1, 4096, 128, 8, W.ZIGZAG, False, 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}P{}{}{}x{}".format(
    c[0], c[1], c[2], c[3], c[4], "csz"[c[5]], "C" if c[6] else "F", c[7]))
def test_backward_parity(case):
    B, H, N, d, P, layout, causal, up = case
    w = W.Workload("bwd", B, H, N, d, P, layout, causal, seed=N + 7 * P, qk_scale_up=up)
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(N + 1)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    got = run_bwd(q, k, v, do, P, layout, causal)
    ref = [np.empty(q.shape) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            rq, rk, rv, _ = OB.attention_backward(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                                  v[b, h].double().numpy(), do[b, h].double().numpy(),
                                                  w.scale, causal)
            ref[0][b, h], ref[1][b, h], ref[2][b, h] = rq, rk, rv
    check(got, ref, str(case))


def test_backward_striped_equals_contiguous():
    """Permutation equivariance of the gradients on the GPU."""
    w = W.Workload("bwd_eq", 1, 2, 2048, 128, 8, W.CONTIGUOUS, True, 11)
    q, k, v = W.make_qkv(w)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    a = run_bwd(q, k, v, do, w.P, W.CONTIGUOUS, True)
    b = run_bwd(q, k, v, do, w.P, W.STRIPED, True)
    for x, y in zip(a, b):
        assert np.abs(x - y).max() <= 2 * REL_MAX * max(np.abs(x).max(), 1e-6)


def test_backward_full_stress_size():
    """The backward at the stress shape (B1 H16 N262144 d128 P16 striped,
    q,k x3): dQ of sampled rows against the oracle's per-row gradient, and
    two identities of the gradients that hold at any size: every row of P
    sums to 1, so sum_j dV_j = sum_i dO_i; every row of dS sums to 0, so
    sum_j dK_j = 0 (per head and dimension; bf16 rounding allowed for)."""
    w = W.STRESS_256K
    q, k, v = W.make_qkv(w)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(12)).to(torch.bfloat16)
    gq, gk, gv = (torch.from_numpy(a) for a in run_bwd(q, k, v, do, w.P, w.layout, w.causal))
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 1, 16383, 16384, 131072, w.N - 1],
                                     rng.integers(0, w.N, 10)]))
    for h in (0, w.H - 1):
        ref = OB.dq_rows(q[0, h].float().numpy(), k[0, h].float().numpy(),
                         v[0, h].float().numpy(), do[0, h].float().numpy(), w.scale, True, rows)
        got = gq[0, h, rows].numpy()
        scale = max(np.abs(ref).max(), 1e-6)
        assert np.abs(got - ref).max() <= REL_MAX * scale, (h, np.abs(got - ref).max() / scale)
    sum_dv = gv[0].double().sum(dim=1)                 # [H, d]
    sum_do = do[0].double().sum(dim=1)
    abs_dv = gv[0].double().abs().sum(dim=1)
    assert torch.all((sum_dv - sum_do).abs() <= 2.0 ** -7 * abs_dv + 1e-3)
    sum_dk = gk[0].double().sum(dim=1)
    abs_dk = gk[0].double().abs().sum(dim=1)
    assert torch.all(sum_dk.abs() <= 2.0 ** -7 * abs_dk + 1e-3)


@pytest.mark.parametrize("layout,N,P", [(W.STRIPED, 2048, 4), (W.ZIGZAG, 4096, 4),
                                        (W.CONTIGUOUS, 1024, 4), (W.STRIPED, 600, 3)])
def test_backward_token_order_is_bit_identical(layout, N, P):
    """RA_TOKEN_ORDER forward + backward on token-order tensors equals the
    partitioned forward + backward, gradients un-partitioned, bit for bit."""
    w = W.Workload("bwd_tok", 1, 2, N, 128, P, layout, True, N + 3, qk_scale_up=3.0)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(N)).to(torch.bfloat16).cuda()
    o_t, l_t = ops.attn_fwd(q, k, v, P, layout, True, token_order=True)
    g_t = ops.attn_bwd(q, k, v, o_t, do, l_t, P, layout, True, token_order=True)
    part = (lambda t: ops.partition(t, P, layout)) if layout != W.CONTIGUOUS else (lambda t: t)
    unpart = ((lambda t: ops.partition(t, P, layout, inverse=True))
              if layout != W.CONTIGUOUS else (lambda t: t))
    qp, kp, vp, dop = (part(t) for t in (q, k, v, do))
    o_p, l_p = ops.attn_fwd(qp, kp, vp, P, layout, True)
    g_p = [unpart(g) for g in ops.attn_bwd(qp, kp, vp, o_p, dop, l_p, P, layout, True)]
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    for a, b in zip(g_t, g_p):
        assert torch.equal(a, b)
