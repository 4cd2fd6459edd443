"""Failure detection on the GPU without a fault: bounded waits that run out.

The self-test kernel waits on a barrier that nothing completes; the wait
gives up after a short limit, the kernel records a fault code and returns.
The attention kernel's own abort path is exercised the same way: its first
S-ready signal is withheld, so a main-loop wait runs out and every role of
every CTA must stop, drain its own MMAs and TMA loads and free its tensor
memory.  The host reads the code, and the context stays usable for real
work (checked against the oracle)."""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import attention as OA

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


def test_wait_that_runs_out_reports_and_context_survives():
    ops.wait_selftest(limit_ns=50_000_000)          # 50 ms
    code = ops.device_fault()
    assert code == 2
    assert ops.device_fault() == 0                   # the word was cleared
    # the context still computes correctly afterwards
    w = W.Workload("after_fault", 1, 1, 512, 64, 2, W.STRIPED, True, 3)
    q, k, v = W.make_qkv(w)
    dq, dk, dv = (ops.partition(t.cuda(), w.P, w.layout) for t in (q, k, v))
    o, lse = ops.attn_fwd(dq, dk, dv, w.P, w.layout, True)
    o = ops.partition(o, w.P, w.layout, inverse=True)
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    o_ref, _ = OA.attention(q[0, 0].double().numpy(), k[0, 0].double().numpy(),
                            v[0, 0].double().numpy(), w.scale, True)
    assert np.abs(o[0, 0].float().cpu().numpy() - o_ref).max() <= 2e-2


def test_selftest_rejects_bad_limit():
    with pytest.raises(ops.RingAttnError):
        ops.wait_selftest(limit_ns=10)


@pytest.mark.parametrize("layout,d", [(W.STRIPED, 128), (W.CONTIGUOUS, 64)])
def test_attention_abort_path_drains_and_context_survives(layout, d):
    w = W.Workload("abort", 1, 4, 8192, d, 4, layout, True, 5, qk_scale_up=3.0)
    q, k, v = W.make_qkv(w)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    if layout != W.CONTIGUOUS:
        dq, dk, dv = (ops.partition(t, w.P, layout) for t in (dq, dk, dv))
    assert ops.device_fault() == 0
    ops.attn_abort_selftest(dq, dk, dv, w.P, layout, True, limit_ns=2_000_000)   # 2 ms
    assert ops.device_fault() == 1
    assert ops.device_fault() == 0
    # twice in a row: nothing the first abort left behind (tensor memory,
    # barriers, loads in flight) may affect the next launch
    ops.attn_abort_selftest(dq, dk, dv, w.P, layout, True, limit_ns=2_000_000)
    assert ops.device_fault() == 1
    o, lse = ops.attn_fwd(dq, dk, dv, w.P, layout, True)
    if layout != W.CONTIGUOUS:
        o = ops.partition(o, w.P, layout, inverse=True)
        lse = ops.partition(lse, w.P, layout, inverse=True)
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    for h in (0, w.H - 1):
        o_ref, lse_ref = OA.attention(q[0, h].double().numpy(), k[0, h].double().numpy(),
                                      v[0, h].double().numpy(), w.scale, True)
        err = np.abs(o[0, h].float().cpu().numpy() - o_ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3
        assert np.abs(lse[0, h].cpu().numpy() - lse_ref).max() <= 1e-3
