"""GPU parity of the CTA-pair forward (RA_CTA_PAIR: clusters of two CTAs
sharing each M = 256 tensor-core MMA, each SM loading half of every
key/value tile) against the fp64 oracle, and against the single-CTA kernel
on the same inputs."""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from tests.test_gpu_parity import assert_close, oracle_full, sample_rows
from oracle import attention as OA

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    assert ops.device_fault() == 0


def run(q, k, v, P, layout, causal, sched_free, pair, o_f32=False):
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    if layout != W.CONTIGUOUS:
        dq, dk, dv = (ops.partition(t, P, layout) for t in (dq, dk, dv))
    o, lse = ops.attn_fwd(dq, dk, dv, P, layout, causal, sched_free=sched_free, cta_pair=pair,
                          o_f32=o_f32)
    if layout != W.CONTIGUOUS:
        o = ops.partition(o, P, layout, inverse=True)
        lse = ops.partition(lse, P, layout, inverse=True)
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


CASES = [
    # (B, H, N, d, P, layout, causal, qk_scale_up)
    (1, 2, 2048, 128, 4, W.STRIPED, True, 3.0),
    (2, 3, 1024, 128, 4, W.CONTIGUOUS, True, 1.0),
    (1, 2, 600, 128, 3, W.STRIPED, True, 1.0),        # c = 200: ragged tiles, a partial quad
    (1, 2, 600, 128, 3, W.CONTIGUOUS, True, 3.0),
    (1, 2, 4096, 128, 16, W.STRIPED, True, 3.0),      # c = 256: one half-filled quad per shard
    (1, 2, 2048, 128, 2, W.STRIPED, False, 1.0),
    (1, 1, 1, 128, 1, W.CONTIGUOUS, True, 1.0),
    (1, 2, 5120, 128, 5, W.STRIPED, True, 3.0),       # c = 1024: two full quads per shard
    (3, 1, 384, 128, 3, W.STRIPED, True, 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}P{}{}{}x{}".format(
    c[0], c[1], c[2], c[3], c[4], "s" if c[5] else "c", "C" if c[6] else "F", c[7]))
@pytest.mark.parametrize("sched_free", [False, True])
def test_pair_parity(case, sched_free):
    B, H, N, d, P, layout, causal, up = case
    w = W.Workload("pair", B, H, N, d, P, layout, causal, seed=N + P + 5, qk_scale_up=up)
    q, k, v = W.make_qkv(w)
    o, lse = run(q, k, v, P, layout, causal, sched_free, True)
    o_ref, lse_ref = oracle_full(q, k, v, causal, w.scale)
    assert_close(o, lse, o_ref, lse_ref, f"pair {case}")
    o1, lse1 = run(q, k, v, P, layout, causal, sched_free, False)
    assert np.abs(o - o1).max() <= 2e-2 and np.abs(lse - lse1).max() <= 1e-3


@pytest.mark.parametrize("w", [W.STRIPED_8K, W.LONG_128K], ids=lambda w: w.name)
def test_pair_workloads_sampled(w):
    q, k, v = W.make_qkv(w)
    o, lse = run(q, k, v, w.P, w.layout, w.causal, False, True)
    for h in (0, w.H - 1):
        rows = sample_rows(w, 24, h)
        o_ref, lse_ref = OA.attention_rows(q[0, h].float().numpy(), k[0, h].float().numpy(),
                                           v[0, h].float().numpy(), w.scale, True, rows)
        assert_close(o[0, h, rows], lse[0, h, rows], o_ref, lse_ref, f"pair {w.name} h{h}")
    assert np.array_equal(o[0, :, 0], v[0, :, 0].float().numpy())


def test_pair_float32_output_rounds_to_bf16_output():
    """RA_O_F32 with the pair kernel: the float32 O rounds to the bf16 O bit
    for bit, and matches the single-CTA kernel's float32 O."""
    w = W.Workload("pair_f32", 1, 2, 2048, 128, 4, W.STRIPED, True, seed=77, qk_scale_up=3.0)
    q, k, v = W.make_qkv(w)
    o32, lse32 = run(q, k, v, w.P, w.layout, True, False, True, o_f32=True)
    o16, lse16 = run(q, k, v, w.P, w.layout, True, False, True)
    rounded = torch.from_numpy(o32).to(torch.bfloat16).float().numpy()
    assert np.array_equal(rounded, o16) and np.array_equal(lse32, lse16)
    o32s, _ = run(q, k, v, w.P, w.layout, True, False, False, o_f32=True)
    assert np.abs(o32 - o32s).max() <= 1e-3
