"""The zigzag layout on the GPU (a reading: the pages only name it; shard j
holds chunks j and 2P-1-j of 2P chunks).  Partition bit-exact against the
oracle's placement, the forward against the plain definition with the
forward's tolerances, the three layouts agreeing after un-partitioning,
stripe + RoPE, and the host-buffer path."""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import attention as OA
from oracle import partition as OP
from oracle import rope as OR
from tests.test_gpu_parity import assert_close, oracle_full, run_path

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    ops.device_fault()


@pytest.mark.parametrize("N,P", [(16, 4), (600, 3), (4096, 8), (4096, 1)])
def test_zigzag_partition_bit_exact(N, P):
    x = torch.randn(2, 3, N, 128, generator=torch.Generator().manual_seed(N)).to(torch.bfloat16)
    y = ops.partition(x.cuda(), P, W.ZIGZAG)
    z = ops.partition(y, P, W.ZIGZAG, inverse=True)
    ref = OP.partition(x.view(torch.int16).numpy(), P, OP.ZIGZAG, axis=2)
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), ref)
    assert torch.equal(z.cpu(), x)
    pos = ops.partition(torch.arange(N, dtype=torch.int32).cuda(), P, W.ZIGZAG).cpu().numpy()
    assert np.array_equal(pos, OP.slot_to_token(N, P, OP.ZIGZAG))


CASES = [
    # (B, H, N, d, P, causal, qk_scale_up)
    (1, 2, 4096, 128, 4, True, 1.0),
    (1, 2, 4096, 128, 4, True, 3.0),
    (2, 1, 2048, 64, 2, True, 1.0),
    (1, 2, 4096, 128, 8, False, 1.0),
    (1, 1, 1024, 128, 2, True, 1.0),         # c = 512: one chunk pair per tile pair
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}P{}{}x{}".format(
    c[0], c[1], c[2], c[3], c[4], "C" if c[5] else "F", c[6]))
@pytest.mark.parametrize("sched_free", [False, True])
def test_zigzag_forward_parity(case, sched_free):
    B, H, N, d, P, causal, up = case
    w = W.Workload("zz", B, H, N, d, P, W.ZIGZAG, causal, seed=N + P, qk_scale_up=up)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, P, W.ZIGZAG, causal, sched_free=sched_free)
    o_ref, lse_ref = oracle_full(q, k, v, causal, w.scale)
    assert_close(o, lse, o_ref, lse_ref, str(case))


def test_three_layouts_agree():
    w = W.Workload("zz_eq", 1, 2, 8192, 128, 8, W.ZIGZAG, True, 9)
    q, k, v = W.make_qkv(w)
    outs = [run_path(q, k, v, w.P, lay, True) for lay in (W.CONTIGUOUS, W.STRIPED, W.ZIGZAG)]
    for o, lse in outs[1:]:
        assert np.abs(o - outs[0][0]).max() <= 4e-2
        assert np.abs(lse - outs[0][1]).max() <= 2e-3


def test_zigzag_long_sampled_rows():
    """c = 16384, P = 16: rows sampled across both chunks of several shards."""
    w = W.Workload("zz_long", 1, 1, 262144, 128, 16, W.ZIGZAG, True, 4, qk_scale_up=3.0)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, W.ZIGZAG, True)
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 1, 8191, 8192, 131071, 131072, w.N - 1],
                                     rng.integers(0, w.N, 64)]))
    ro, rl = OA.attention_rows(q[0, 0].float().numpy(), k[0, 0].float().numpy(),
                               v[0, 0].float().numpy(), w.scale, True, rows)
    err = np.abs(o[0, 0, rows] - ro)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert np.abs(lse[0, 0, rows] - rl).max() <= 1e-3


def test_zigzag_rope_and_host_path():
    w = W.Workload("zz_host", 1, 3, 2048, 128, 2, W.ZIGZAG, True, 5)
    q, k, v = W.make_qkv(w)
    got = ops.partition_rope(q.cuda(), w.P, W.ZIGZAG, 10000.0, ops.ROPE_HALF).float().cpu().numpy()
    ref = OR.rope_partition(q.double().numpy(), w.P, OP.ZIGZAG, 10000.0, OR.HALF)
    assert np.all(np.abs(got - ref) <= 2.0 ** -7 * np.maximum(np.abs(ref), 2.0 ** -8))
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    ws = torch.empty(ops.attn_fwd_host_workspace_bytes(w.N, w.d, W.ZIGZAG, 1), dtype=torch.uint8,
                     device="cuda")
    o, lse = ops.attn_fwd_host(hq, hk, hv, w.P, W.ZIGZAG, True, workspace=ws)
    torch.cuda.synchronize()
    o_ref, lse_ref = run_path(q, k, v, w.P, W.ZIGZAG, True)
    assert np.array_equal(o.float().numpy(), o_ref)
    assert np.array_equal(lse.numpy(), lse_ref)
