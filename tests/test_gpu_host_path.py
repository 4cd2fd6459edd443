"""ra_attn_fwd_host (host buffers in and out, head chunks pipelined against
the copies) gives bit-identical results to the device path (ra_partition +
ra_attn_fwd + inverse ra_partition): every (b, h) is computed alone, so
chunking changes nothing."""

import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


def device_path(q, k, v, P, layout, causal):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    if layout == W.STRIPED:
        qd, kd, vd = (ops.partition(t, P, layout) for t in (qd, kd, vd))
    o, lse = ops.attn_fwd(qd, kd, vd, P, layout, causal)
    if layout == W.STRIPED:
        o = ops.partition(o, P, layout, inverse=True)
        lse = ops.partition(lse, P, layout, inverse=True)
    return o.cpu(), lse.cpu()


CASES = [
    # (B, H, N, d, P, layout, causal, heads per chunk)
    (1, 16, 8192, 128, 8, W.STRIPED, True, 4),
    (2, 3, 1200, 128, 3, W.STRIPED, True, 1),
    (1, 5, 2048, 64, 4, W.CONTIGUOUS, True, 2),
    (1, 2, 1024, 128, 2, W.STRIPED, False, 8),
    (1, 7, 2048, 128, 4, W.STRIPED, True, 4),      # chunks of 1, 2, 2, 1, 1 heads
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}P{}{}{}G{}".format(
    c[0], c[1], c[2], c[3], c[4], "s" if c[5] else "c", "C" if c[6] else "F", c[7]))
def test_host_path_is_bit_identical_to_device_path(case):
    B, H, N, d, P, layout, causal, G = case
    w = W.Workload("host", B, H, N, d, P, layout, causal, seed=N + H)
    q, k, v = (t.pin_memory() for t in W.make_qkv(w))
    ws = torch.empty(ops.attn_fwd_host_workspace_bytes(N, d, layout, G), dtype=torch.uint8,
                     device="cuda")
    for _ in range(2):                      # the second call reuses streams and workspace
        o, lse = ops.attn_fwd_host(q, k, v, P, layout, causal, workspace=ws)
        torch.cuda.synchronize()
        assert ops.device_fault() == 0
        o_ref, lse_ref = device_path(q, k, v, P, layout, causal)
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, lse_ref)


def test_host_path_rejects_small_workspace():
    w = W.Workload("host_small", 1, 2, 1024, 128, 4, W.STRIPED, True, 3)
    q, k, v = W.make_qkv(w)
    need = ops.attn_fwd_host_workspace_bytes(1024, 128, W.STRIPED, 1)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.RingAttnError) as e:
        ops.attn_fwd_host(q, k, v, 4, W.STRIPED, True, workspace=ws)
    assert e.value.status == 14
