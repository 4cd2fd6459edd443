"""GPU parity of ra_partition_rope (stripe + rotary embedding at original
positions) against the oracle, and RoPE'd striped attention end to end.

The kernel evaluates angles in double precision, rotates in fp32 and rounds
to bf16 once; the oracle rotates in fp64.  Bar: every element within one
bf16 rounding step of the oracle's value (half an ulp for the final
rounding plus the fp32 rotation error, so 1 ulp of max(|ref|, 2^-10 |row|)),
and at least 99 % of the elements bit-identical to the oracle rounded to
bf16 (round to nearest even).
"""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import attention as OA
from oracle import partition as OP
from oracle import rope as OR

pytestmark = pytest.mark.gpu

PAIRING = {ops.ROPE_INTERLEAVED: OR.INTERLEAVED, ops.ROPE_HALF: OR.HALF}
LAYOUT = {W.CONTIGUOUS: OP.CONTIGUOUS, W.STRIPED: OP.STRIPED}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()


def bf16_ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - 7)


def check_rope(got, ref, what):
    got = got.astype(np.float64)
    row = np.abs(ref).max(axis=-1, keepdims=True)
    mag = np.maximum(np.abs(ref), row * 2.0 ** -10)
    err = np.abs(got - ref)
    assert np.all(err <= bf16_ulp(mag)), f"{what}: max err/ulp {np.max(err / bf16_ulp(mag)):.2f}"
    exact = torch.from_numpy(ref).to(torch.bfloat16).float().numpy()
    frac = np.mean(got == exact)
    assert frac >= 0.99, f"{what}: only {frac:.4f} bit-identical"


CASES = [
    # (B, H, N, d, P, layout, pairing, base)
    (1, 2, 1000, 128, 5, W.STRIPED, ops.ROPE_INTERLEAVED, 10000.0),
    (2, 1, 1024, 64, 4, W.CONTIGUOUS, ops.ROPE_HALF, 10000.0),
    (1, 3, 4096, 128, 8, W.STRIPED, ops.ROPE_HALF, 500000.0),
    (1, 1, 48, 16, 3, W.STRIPED, ops.ROPE_INTERLEAVED, 10.0),
    (1, 1, 96, 256, 2, W.STRIPED, ops.ROPE_HALF, 10000.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}N{}d{}P{}{}{}b{:g}".format(
    c[0], c[1], c[2], c[3], c[4], "s" if c[5] else "c", "h" if c[6] else "i", c[7]))
def test_partition_rope_parity(case):
    B, H, N, d, P, layout, pairing, base = case
    x = torch.randn(B, H, N, d, generator=torch.Generator().manual_seed(N + d)).to(torch.bfloat16)
    got = ops.partition_rope(x.cuda(), P, layout, base, pairing).float().cpu().numpy()
    ref = OR.rope_partition(x.double().numpy(), P, LAYOUT[layout], base, PAIRING[pairing])
    check_rope(got, ref, str(case))


def test_partition_rope_long_sequence_sampled_rows():
    """N = 262144 (angles up to 2.6e5 rad): rows sampled across the sequence."""
    B, H, N, d, P = 1, 1, 262144, 128, 16
    x = torch.randn(B, H, N, d, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    got = ops.partition_rope(x.cuda(), P, W.STRIPED, 10000.0, ops.ROPE_HALF).float().cpu().numpy()
    rng = np.random.default_rng(0)
    tokens = np.unique(np.concatenate([[0, 1, N - 1, N - P], rng.integers(0, N, 2000)]))
    slot_of = np.argsort(OP.slot_to_token(N, P, OP.STRIPED))
    ref = OR.rope(x[0, 0, tokens].double().numpy(), tokens, 10000.0, OR.HALF)
    check_rope(got[0, 0, slot_of[tokens]], ref, "N262144")


def test_rope_striped_attention_end_to_end():
    """RoPE'd q, k striped by ra_partition_rope, v by ra_partition, striped
    causal attention, un-partitioned: equals the oracle's attention of the
    RoPE'd tensors in token order (the position encoding survives the
    stripe)."""
    w = W.Workload("rope_e2e", 1, 2, 2048, 128, 8, W.STRIPED, True, 21)
    q, k, v = W.make_qkv(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    qs = ops.partition_rope(qd, w.P, w.layout, 10000.0, ops.ROPE_HALF)
    ks = ops.partition_rope(kd, w.P, w.layout, 10000.0, ops.ROPE_HALF)
    vs = ops.partition(vd, w.P, w.layout)
    o, lse = ops.attn_fwd(qs, ks, vs, w.P, w.layout, True)
    o = ops.partition(o, w.P, w.layout, inverse=True).float().cpu().numpy()
    pos = np.arange(w.N)
    for h in range(w.H):
        qr = OR.rope(q[0, h].double().numpy(), pos, 10000.0, OR.HALF)
        kr = OR.rope(k[0, h].double().numpy(), pos, 10000.0, OR.HALF)
        # the kernel consumes the bf16-rounded rotation
        qr = torch.from_numpy(qr).to(torch.bfloat16).double().numpy()
        kr = torch.from_numpy(kr).to(torch.bfloat16).double().numpy()
        ref, _ = OA.attention(qr, kr, v[0, h].double().numpy(), w.scale, True)
        err = np.abs(o[0, h] - ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (h, err.max(), err.mean())
