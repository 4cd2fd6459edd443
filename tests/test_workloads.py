"""The seeded input generators: determinism and per-head drawing."""

import torch

from long_context_exact_attn_b200 import workloads as W


def test_head_draw_matches_full_draw():
    w = W.Workload("t", 2, 3, 64, 16, 4, W.STRIPED, True, 11, qk_scale_up=3.0)
    q, k, v = W.make_qkv(w)
    for b in range(2):
        for h in range(3):
            qh, kh, vh = W.make_qkv_head(w, b, h)
            assert torch.equal(qh, q[b, h]) and torch.equal(kh, k[b, h]) and torch.equal(vh, v[b, h])


def test_inputs_are_bf16_and_seeded():
    q1, _, _ = W.make_qkv(W.TINY)
    q2, _, _ = W.make_qkv(W.TINY)
    assert q1.dtype == torch.bfloat16 and torch.equal(q1, q2)
    assert tuple(q1.shape) == (1, 1, 256, 64)


def test_useful_flops():
    assert W.RING_8K.useful_pairs() == 8192 * 8193 // 2
    assert W.STRESS_256K.useful_flops() == 4 * 128 * 16 * (262144 * 262145 // 2)
    assert W.TINY.useful_pairs() == 256 * 256
