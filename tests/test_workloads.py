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


def test_useful_pairs_equal_the_oracles_per_round_counts():
    """The bench's FLOP count (4 d per unmasked pair) rests on useful_pairs;
    summed over shards and rounds, the oracle's brute-force counts from
    token positions give the same number for every workload's layout,
    causality and P (at a shard length of 8)."""
    from oracle import partition as OP
    from oracle import work
    lay = {W.CONTIGUOUS: OP.CONTIGUOUS, W.STRIPED: OP.STRIPED, W.ZIGZAG: OP.ZIGZAG}
    for w in W.ALL:
        small = w.with_(N=w.P * 8)
        total = sum(work.work_brute_force(j, r, small.N, small.P, lay[small.layout],
                                          small.causal)
                    for j in range(small.P) for r in range(small.P))
        assert total == small.useful_pairs(), w.name
    zz = W.STRIPED_8K.with_(layout=W.ZIGZAG, N=4 * 8, P=4)
    assert sum(work.work_brute_force(j, r, zz.N, zz.P, OP.ZIGZAG, True)
               for j in range(4) for r in range(4)) == zz.useful_pairs()
