"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The self-test kernel waits on a barrier that nothing completes; the wait
gives up after a short limit, the kernel records a fault code and returns.
The host reads the code, and the context stays usable for real work."""

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
