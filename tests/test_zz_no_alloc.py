"""ra_attn_bwd_noalloc: the backward without a caller workspace.

Runs on the GPU through the C-ABI and compares the allocation-free entry point
with ra_attn_bwd (same inputs, caller workspace) on two calls in a row, each
within the backward tolerance of the parity tests: max |g - g_ref| <= 2e-2 *
max|g_ref| and mean |g - g_ref| <= 2e-3 * max|g_ref| per tensor.  The two
paths run the same kernels, so in practice they agree bit for bit; each call's
gradients are therefore also checked against the fp64 oracle's gradients of
the plain definition, so that an error common to both paths would show.  The
second call uses other inputs, so stale contents of the shared scratch from
the first call would show.
"""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import backward as OB

pytestmark = pytest.mark.gpu

REL_MAX, REL_MEAN = 2e-2, 2e-3
MAX_ROWS = 1 << 20


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


def _inputs(w, seed):
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16).cuda()
    q, k, v, do = (ops.partition(t, w.P, w.layout) for t in (q, k, v, do))
    o, lse = ops.attn_fwd(q, k, v, w.P, w.layout, w.causal)
    return q, k, v, o, do, lse


def _oracle_grads(w, do_seed):
    """The fp64 oracle's dQ, dK, dV of the same token-order inputs."""
    q, k, v = W.make_qkv(w)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(do_seed)).to(torch.bfloat16)
    out = [np.empty(q.shape) for _ in range(3)]
    for b in range(w.B):
        for h in range(w.H):
            g = OB.attention_backward(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                      v[b, h].double().numpy(), do[b, h].double().numpy(),
                                      w.scale, w.causal)
            for t in range(3):
                out[t][b, h] = g[t]
    return out


def _close(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g, r = g.float().cpu().numpy(), r.float().cpu().numpy()
        scale = max(np.abs(r).max(), 1e-6)
        err = np.abs(g - r)
        assert np.isfinite(g).all(), f"{what} {name}"
        assert err.max() <= REL_MAX * scale, f"{what} {name}: max {err.max() / scale:.3e}"
        assert err.mean() <= REL_MEAN * scale, f"{what} {name}: mean {err.mean() / scale:.3e}"


def test_noalloc_matches_workspace_backward_twice():
    cases = [W.Workload("noalloc_a", 1, 2, 2048, 128, 4, W.STRIPED, True, 31),
             W.Workload("noalloc_b", 2, 1, 1500, 64, 5, W.STRIPED, True, 32, qk_scale_up=3.0)]
    for call, w in enumerate(cases):
        q, k, v, o, do, lse = _inputs(w, 100 + call)
        ref = ops.attn_bwd(q, k, v, o, do, lse, w.P, w.layout, w.causal, w.scale)
        got = [torch.empty_like(q) for _ in range(3)]
        ops.attn_bwd_noalloc(q, k, v, o, do, lse, w.P, w.layout, w.causal, w.scale, *got)
        torch.cuda.synchronize()
        assert ops.device_fault() == 0
        _close(got, ref, f"call {call} ({w.name})")
        tok = [ops.partition(g, w.P, w.layout, inverse=True) for g in got]
        _close(tok, [torch.from_numpy(a) for a in _oracle_grads(w, 100 + call)],
               f"call {call} ({w.name}) against the oracle")


def test_noalloc_rejects_more_rows_than_its_scratch():
    # B*H*N one tile past the built-in maximum; nothing may be launched.
    N = MAX_ROWS // 4 + 128
    q = torch.zeros(1, 4, N, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 4, N, dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(q) for _ in range(3)]
    with pytest.raises(ops.RingAttnError) as e:
        ops.attn_bwd_noalloc(q, q.clone(), q.clone(), q.clone(), q.clone(), lse, 1,
                             W.CONTIGUOUS, True, 0.125, *outs)
    assert e.value.status == 12
