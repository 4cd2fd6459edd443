"""GPU parity of the ring's per-round step (ra_attn_fwd_block) and of the
ring emulated on one device (every rank's rounds in turn: ra_attn_fwd_block
+ ra_lse_merge_acc) against the oracle.

Tolerances as the forward: O max-abs 2e-2, mean-abs 2e-3 against fp64; lse
1e-3 where a row sees a key; rows that see no key of a block must be
exactly (0, -inf).
"""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import attention as OA
from oracle import partition as OP
from oracle import ring as OR

pytestmark = pytest.mark.gpu

LAY = {W.CONTIGUOUS: OP.CONTIGUOUS, W.STRIPED: OP.STRIPED}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


def _layout_qkv(w):
    q, k, v = W.make_qkv(w)
    return [ops.partition(t.cuda(), w.P, w.layout) for t in (q, k, v)]


BLOCK_CASES = [
    # (H, N, d, P, layout, causal, qk_scale_up)
    (2, 1024, 128, 4, W.STRIPED, True, 3.0),
    (2, 1024, 128, 4, W.CONTIGUOUS, True, 1.0),
    (1, 600, 64, 3, W.STRIPED, True, 1.0),       # ragged shards
    (1, 512, 128, 2, W.STRIPED, False, 1.0),
    (1, 8, 128, 8, W.STRIPED, True, 1.0),        # c = 1: rows with no key
    (1, 24, 64, 4, W.CONTIGUOUS, True, 1.0),     # hidden blocks, tiny shards
]


@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: "H{}N{}d{}P{}{}{}x{}".format(
    c[0], c[1], c[2], c[3], "s" if c[4] else "c", "C" if c[5] else "F", c[6]))
def test_block_parity_all_pairs(case):
    H, N, d, P, layout, causal, up = case
    w = W.Workload("blk", 1, H, N, d, P, layout, causal, seed=N + P, qk_scale_up=up)
    qp, kp, vp = _layout_qkv(w)
    c = N // P
    sh = lambda t, j: t[:, :, j * c:(j + 1) * c].contiguous()
    for j in range(P):
        for kb in range(P):
            o, lse = ops.attn_fwd_block(sh(qp, j), sh(kp, kb), sh(vp, kb), j, kb, P, layout, causal)
            o32, lse32 = ops.attn_fwd_block(sh(qp, j), sh(kp, kb), sh(vp, kb), j, kb, P, layout,
                                            causal, o_f32=True)
            torch.cuda.synchronize()
            # the float32 partial is the same O before its rounding
            assert o32.dtype == torch.float32 and torch.equal(o32.to(torch.bfloat16), o)
            assert torch.equal(lse32, lse)
            o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
            for h in range(H):
                ro, rl = OR.block_attention(sh(qp, j)[0, h].double().cpu().numpy(),
                                            sh(kp, kb)[0, h].double().cpu().numpy(),
                                            sh(vp, kb)[0, h].double().cpu().numpy(),
                                            j, kb, P, LAY[layout], causal, w.scale)
                empty = np.isneginf(rl)
                assert np.array_equal(np.isneginf(lse[0, h]), empty), (j, kb, h)
                assert np.all(o[0, h][empty] == 0), (j, kb, h)
                err = np.abs(o[0, h] - ro)
                assert err.max() <= 2e-2 and err.mean() <= 2e-3, (j, kb, h, err.max())
                if (~empty).any():
                    assert np.abs(lse[0, h][~empty] - rl[~empty]).max() <= 1e-3, (j, kb, h)
    assert ops.device_fault() == 0


@pytest.mark.parametrize("layout,P", [(W.STRIPED, 8), (W.CONTIGUOUS, 8), (W.CONTIGUOUS, 4),
                                      (W.STRIPED, 4)])
def test_emulated_ring_equals_fused_forward_and_definition(layout, P):
    """Each rank j folds block (j - r) mod P in round r (Ring explainer
    ステップ2) through the float32 accumulator, with float32 partials (O is
    rounded to bf16 once); the result equals the fused single-launch forward
    and the plain definition."""
    w = W.Workload("ring_emu", 1, 2, 4096 if P == 8 else 2048, 128, P, layout, True, 77 + P,
                   qk_scale_up=3.0)
    qp, kp, vp = _layout_qkv(w)
    P, c = w.P, w.N // w.P
    o_fused, lse_fused = ops.attn_fwd(qp, kp, vp, P, layout, True)
    o_ring = torch.empty_like(qp)
    lse_ring = torch.empty(1, w.H, w.N, device="cuda")
    for j in range(P):
        q = qp[:, :, j * c:(j + 1) * c].contiguous()
        acc = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        lacc = torch.empty(1, w.H, c, device="cuda")
        out = torch.empty_like(q)
        for r in range(P):
            kb = (j - r) % P
            o_r, l_r = ops.attn_fwd_block(q, kp[:, :, kb * c:(kb + 1) * c].contiguous(),
                                          vp[:, :, kb * c:(kb + 1) * c].contiguous(), j, kb, P,
                                          layout, True, o_f32=True)
            ops.lse_merge_acc(acc, lacc, o_r, l_r, first=(r == 0),
                              final_out=out if r == P - 1 else None)
        o_ring[:, :, j * c:(j + 1) * c] = out
        lse_ring[:, :, j * c:(j + 1) * c] = lacc
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    o_ring_t = ops.partition(o_ring, P, layout, inverse=True).float().cpu().numpy()
    lse_ring_t = ops.partition(lse_ring, P, layout, inverse=True).cpu().numpy()
    o_fused_t = ops.partition(o_fused, P, layout, inverse=True).float().cpu().numpy()
    q, k, v = W.make_qkv(w)
    for h in range(w.H):
        ro, rl = OA.attention(q[0, h].double().numpy(), k[0, h].double().numpy(),
                              v[0, h].double().numpy(), w.scale, True)
        err = np.abs(o_ring_t[0, h] - ro)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (h, err.max(), err.mean())
        assert np.abs(lse_ring_t[0, h] - rl).max() <= 1e-3
        assert np.abs(o_ring_t[0, h] - o_fused_t[0, h]).max() <= 4e-2
