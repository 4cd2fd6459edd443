"""A seeded sweep of shapes against the oracle: shard lengths from 1 to
several tiles (ragged ones included), P from 1 to N, d 64 and 128, all three
layouts (zigzag where N/P is a multiple of 512), causal and not, q,k x1 and
x3, one or two batch entries.  Per case: the forward (partitioned path) within the forward tolerances,
the token-order path bit-identical to it, and for every third case the
backward within its tolerances."""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import backward as OB
from tests.test_gpu_parity import assert_close, oracle_full, run_path

pytestmark = pytest.mark.gpu


def _cases(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        P = int(rng.choice([1, 2, 3, 5, 8, 16]))
        c = int(rng.choice([1, 7, 64, 127, 128, 129, 200, 256, 384, 512, 700]))
        layout = int(rng.choice([W.CONTIGUOUS, W.STRIPED, W.ZIGZAG]))
        if layout == W.ZIGZAG:
            c = 512 * int(rng.integers(1, 3))
            P = int(rng.choice([1, 2, 4]))
        N = c * P
        d = int(rng.choice([64, 128]))
        causal = bool(rng.random() < 0.8)
        up = float(rng.choice([1.0, 3.0]))
        H = int(rng.choice([1, 2]))
        B = int(rng.choice([1, 2])) if N <= 4096 else 1
        out.append((i, B, H, N, d, P, layout, causal, up))
    return out


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


@pytest.mark.parametrize("case", _cases(), ids=lambda c: "i{}B{}H{}N{}d{}P{}{}{}x{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], "csz"[c[6]], "C" if c[7] else "F", c[8]))
def test_sweep(case):
    i, B, H, N, d, P, layout, causal, up = case
    w = W.Workload("sweep", B, H, N, d, P, layout, causal, seed=1000 + i, qk_scale_up=up)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, P, layout, causal)
    o_ref, lse_ref = oracle_full(q, k, v, causal, w.scale)
    assert_close(o, lse, o_ref, lse_ref, str(case))
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o_t, l_t = ops.attn_fwd(qd, kd, vd, P, layout, causal, token_order=True)
    torch.cuda.synchronize()
    assert np.array_equal(o_t.float().cpu().numpy(), o)
    assert np.array_equal(l_t.cpu().numpy(), lse)
    if i % 3 == 0:
        do = torch.randn(q.shape, generator=torch.Generator().manual_seed(i)).to(torch.bfloat16)
        grads = ops.attn_bwd(qd, kd, vd, o_t, do.cuda(), l_t, P, layout, causal, token_order=True)
        torch.cuda.synchronize()
        assert ops.device_fault() == 0
        for b, h in ((b, h) for b in range(B) for h in range(H)):
            ref = OB.attention_backward(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                        v[b, h].double().numpy(), do[b, h].double().numpy(),
                                        w.scale, causal)[:3]
            for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
                g = g[b, h].float().cpu().numpy()
                scale = max(np.abs(r).max(), 1e-6)
                err = np.abs(g - r)
                assert err.max() <= 2e-2 * scale, (case, name, err.max() / scale)
                assert err.mean() <= 2e-3 * scale, (case, name, err.mean() / scale)
