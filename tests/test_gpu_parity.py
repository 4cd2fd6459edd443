"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output), against the fp64
oracle on the same bf16 inputs: O max-abs <= 2e-2 and mean-abs <= 2e-3;
lse max-abs <= 1e-3.  Integer results (permutations, tile counts, visible
pairs) must match exactly.
"""

import numpy as np
import pytest
import torch

from long_context_exact_attn_b200 import ops
from long_context_exact_attn_b200 import workloads as W
from oracle import attention as OA
from oracle import merge as OM
from oracle import partition as OP
from oracle import work as OW
from tests import _margins

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
LAYOUT = {W.CONTIGUOUS: OP.CONTIGUOUS, W.STRIPED: OP.STRIPED, W.ZIGZAG: OP.ZIGZAG}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    assert ops.device_fault() == 0


def run_path(q, k, v, P, layout, causal, sched_free=False, scale=None):
    """The whole hot path on the GPU: partition -> attention -> un-partition.
    q, k, v: CPU bf16 [B, H, N, d] in token order.  Returns O (float32 numpy,
    token order) and lse (numpy, token order)."""
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    if layout != W.CONTIGUOUS:
        dq, dk, dv = (ops.partition(t, P, layout) for t in (dq, dk, dv))
    o, lse = ops.attn_fwd(dq, dk, dv, P, layout, causal, scale=scale, sched_free=sched_free)
    if layout != W.CONTIGUOUS:
        o = ops.partition(o, P, layout, inverse=True)
        lse = ops.partition(lse, P, layout, inverse=True)
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def oracle_full(q, k, v, causal, scale):
    B, H = q.shape[:2]
    o = np.empty(q.shape[:-1] + (v.shape[-1],))
    lse = np.empty(q.shape[:-1])
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = OA.attention(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                              v[b, h].double().numpy(), scale, causal)
    return o, lse


def assert_close(o, lse, o_ref, lse_ref, what=""):
    err = np.abs(o - o_ref)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), what
    lerr = np.abs(lse - lse_ref)
    _margins.record(what, err.max(), err.mean(), lerr.max())
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3e}"
    assert lerr.max() <= LSE_MAX, f"{what}: lse max-abs {lerr.max():.3e}"


SMALL = [
    # (B, H, N, d, P, layout, causal, qk_scale_up)
    (1, 1, 256, 64, 4, W.CONTIGUOUS, False, 1.0),     # the tiny workload's shape
    (2, 3, 1024, 128, 4, W.CONTIGUOUS, True, 1.0),
    (2, 3, 1024, 128, 4, W.STRIPED, True, 1.0),
    (1, 2, 600, 128, 3, W.STRIPED, True, 1.0),        # c = 200: ragged tiles
    (1, 2, 600, 128, 3, W.CONTIGUOUS, True, 1.0),
    (1, 2, 1500, 64, 5, W.STRIPED, True, 3.0),        # c = 300: odd tile count
    (1, 2, 1500, 64, 5, W.CONTIGUOUS, False, 1.0),
    (1, 1, 2048, 128, 1, W.CONTIGUOUS, True, 3.0),    # one shard = plain causal
    (1, 2, 512, 128, 8, W.STRIPED, True, 1.0),        # c = 64 < tile
    (1, 1, 8, 64, 2, W.STRIPED, True, 1.0),
    (1, 1, 1, 128, 1, W.CONTIGUOUS, True, 1.0),
    (1, 4, 4096, 128, 16, W.STRIPED, True, 3.0),
    (1, 2, 2048, 64, 2, W.STRIPED, False, 1.0),
    (3, 1, 384, 128, 3, W.STRIPED, True, 1.0),        # c = 128: one tile per shard
    (1, 1, 1000, 128, 5, W.STRIPED, True, 3.0),       # c = 200, P not a power of two
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B{}H{}N{}d{}P{}{}{}x{}".format(
    c[0], c[1], c[2], c[3], c[4], "s" if c[5] else "c", "C" if c[6] else "F", c[7]))
@pytest.mark.parametrize("sched_free", [False, True])
def test_parity_small(case, sched_free):
    B, H, N, d, P, layout, causal, up = case
    w = W.Workload("t", B, H, N, d, P, layout, causal, seed=N + P + d, qk_scale_up=up)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, P, layout, causal, sched_free)
    o_ref, lse_ref = oracle_full(q, k, v, causal, w.scale)
    assert_close(o, lse, o_ref, lse_ref, str(case))


def test_tiny_workload_elementwise():
    w = W.TINY
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, w.layout, w.causal)
    o_ref, lse_ref = oracle_full(q, k, v, w.causal, w.scale)
    assert_close(o, lse, o_ref, lse_ref, w.name)


def sample_rows(w, n_random, seed):
    """Row 0, every shard's first and last token (in layout terms), tile
    edges of shard 0, and random rows -- as original token indices."""
    rng = np.random.default_rng(seed)
    perm = OP.slot_to_token(w.N, w.P, LAYOUT[w.layout]) if w.N <= 1 << 18 else None
    slots = {0, w.N - 1}
    for j in range(w.P):
        slots.update({j * w.c, j * w.c + w.c - 1})
    for x in (127, 128, 255, 256):
        if x < w.c:
            slots.add(x)
    slots.update(rng.integers(0, w.N, n_random).tolist())
    return sorted({int(perm[s]) for s in slots})


@pytest.mark.parametrize("w", [W.RING_8K, W.STRIPED_8K], ids=lambda w: w.name)
@pytest.mark.parametrize("sched_free", [False, True])
def test_parity_8k_workloads(w, sched_free):
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, w.layout, w.causal, sched_free)
    for h in (0, w.H - 1):        # whole heads, element by element
        o_ref, lse_ref = OA.attention(q[0, h].double().numpy(), k[0, h].double().numpy(),
                                      v[0, h].double().numpy(), w.scale, True)
        assert_close(o[0, h], lse[0, h], o_ref, lse_ref, f"{w.name} head {h}")
    for h in range(1, w.H - 1):   # sampled rows elsewhere
        rows = sample_rows(w, 16, h)
        o_ref, lse_ref = OA.attention_rows(q[0, h].float().numpy(), k[0, h].float().numpy(), v[0, h].float().numpy(),
                                           w.scale, True, rows)
        assert_close(o[0, h, rows], lse[0, h, rows], o_ref, lse_ref, f"{w.name} head {h}")
    # causal row 0 sees only key 0: O row 0 is v_0 exactly
    assert np.array_equal(o[0, :, 0], v[0, :, 0].float().numpy())


def test_striped_equals_contiguous_on_same_inputs():
    """Permutation equivariance on the GPU: the striped path, un-permuted,
    matches the contiguous path on the same inputs (both within tolerance of
    one oracle, and within twice the tolerance of each other)."""
    w = W.RING_8K.with_(H=4)
    q, k, v = W.make_qkv(w)
    oc, lc = run_path(q, k, v, w.P, W.CONTIGUOUS, True)
    os_, ls = run_path(q, k, v, w.P, W.STRIPED, True)
    assert np.abs(oc - os_).max() <= 2 * O_MAX
    assert np.abs(lc - ls).max() <= 2 * LSE_MAX
    o_ref, lse_ref = oracle_full(q, k, v, True, w.scale)
    assert_close(oc, lc, o_ref, lse_ref, "contiguous")
    assert_close(os_, ls, o_ref, lse_ref, "striped")


def test_constant_v_gives_constant_o():
    w = W.Workload("constv", 1, 2, 2048, 128, 8, W.STRIPED, True, 7, qk_scale_up=3.0)
    q, k, _ = W.make_qkv(w)
    row = torch.randn(128, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    v = row.expand(1, 2, 2048, 128).contiguous()
    o, _ = run_path(q, k, v, w.P, w.layout, True)
    ref = np.broadcast_to(row.float().numpy(), o.shape)
    assert np.abs(o - ref).max() <= O_MAX


@pytest.mark.parametrize("w", [W.LONG_128K, W.STRESS_256K], ids=lambda w: w.name)
@pytest.mark.parametrize("sched_free", [False, True])
def test_parity_long_workloads_sampled(w, sched_free):
    """Full-size long workloads, in the launch configuration the benchmark
    times; sampled rows against the oracle computed row by row."""
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, w.layout, w.causal, sched_free)
    for h in (0, w.H // 2, w.H - 1):
        rows = sample_rows(w, 24, h)
        o_ref, lse_ref = OA.attention_rows(q[0, h].float().numpy(), k[0, h].float().numpy(), v[0, h].float().numpy(),
                                           w.scale, True, rows)
        assert_close(o[0, h, rows], lse[0, h, rows], o_ref, lse_ref, f"{w.name} head {h}")
    assert np.array_equal(o[0, :, 0], v[0, :, 0].float().numpy())
    assert np.isfinite(o).all() and np.isfinite(lse).all()


def test_parity_d64_batched_striped():
    """d = 64 at scale, B > 1, striped causal: two heads element by element,
    sampled rows elsewhere."""
    w = W.Workload("d64", 2, 4, 8192, 64, 8, W.STRIPED, True, 21, qk_scale_up=3.0)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, w.layout, True)
    for b, h in ((0, 0), (1, 3)):
        o_ref, lse_ref = OA.attention(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                      v[b, h].double().numpy(), w.scale, True)
        assert_close(o[b, h], lse[b, h], o_ref, lse_ref, f"d64 b{b} h{h}")
    for b, h in ((0, 2), (1, 1)):
        rows = sample_rows(w, 16, b * 7 + h)
        o_ref, lse_ref = OA.attention_rows(q[b, h].float().numpy(), k[b, h].float().numpy(),
                                           v[b, h].float().numpy(), w.scale, True, rows)
        assert_close(o[b, h, rows], lse[b, h, rows], o_ref, lse_ref, f"d64 b{b} h{h} rows")


def test_parity_noncausal_long_sampled():
    """Non-causal striped, N = 32768: every row attends to every key."""
    w = W.Workload("noncausal32k", 1, 2, 32768, 128, 8, W.STRIPED, False, 22)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, w.layout, False)
    for h in range(2):
        rows = sample_rows(w, 24, h)
        o_ref, lse_ref = OA.attention_rows(q[0, h].float().numpy(), k[0, h].float().numpy(),
                                           v[0, h].float().numpy(), w.scale, False, rows)
        assert_close(o[0, h, rows], lse[0, h, rows], o_ref, lse_ref, f"noncausal h{h}")


def test_parity_long_contiguous_sampled():
    """The contiguous (ring) layout at the 128K size, as the benchmark's
    layout comparison runs it."""
    w = W.LONG_128K.with_(layout=W.CONTIGUOUS)
    q, k, v = W.make_qkv(w)
    o, lse = run_path(q, k, v, w.P, w.layout, True)
    for h in (0, w.H - 1):
        rows = sample_rows(w, 24, h)
        o_ref, lse_ref = OA.attention_rows(q[0, h].float().numpy(), k[0, h].float().numpy(),
                                           v[0, h].float().numpy(), w.scale, True, rows)
        assert_close(o[0, h, rows], lse[0, h, rows], o_ref, lse_ref, f"contiguous 128K h{h}")


# ------------------------------------------------------------ integer parity
@pytest.mark.parametrize("N,P,layout,causal", [
    (8192, 8, W.CONTIGUOUS, True), (8192, 8, W.STRIPED, True), (131072, 8, W.STRIPED, True),
    (262144, 16, W.STRIPED, True), (262144, 16, W.CONTIGUOUS, True), (256, 4, W.CONTIGUOUS, False),
    (4096, 4, W.STRIPED, False)])
def test_tile_census_closed_forms(N, P, layout, causal):
    got = ops.tile_census(N, P, layout, causal).cpu().numpy()
    c = N // P
    for j in range(P):
        for r in range(P):
            if c % 128 == 0:
                exp = OW.tile_census_closed_form(j, r, c, P, LAYOUT[layout], causal, 128)
                assert tuple(got[j, r, :3]) == exp, (j, r)
            assert got[j, r, 3] == OW.work_exact_closed_form(j, r, c, P, LAYOUT[layout], causal)
    assert got[:, :, 3].sum() == (N * (N + 1) // 2 if causal else N * N)


@pytest.mark.parametrize("N,P,layout,causal", [
    (600, 3, W.STRIPED, True), (600, 3, W.CONTIGUOUS, True), (1500, 5, W.STRIPED, True),
    (512, 8, W.STRIPED, True), (1024, 4, W.CONTIGUOUS, True), (768, 2, W.STRIPED, False)])
def test_tile_census_brute_force(N, P, layout, causal):
    got = ops.tile_census(N, P, layout, causal).cpu().numpy()
    for j in range(P):
        for r in range(P):
            exp = OW.tile_census_brute_force(j, r, N, P, LAYOUT[layout], causal, 128, 128)
            assert tuple(int(x) for x in got[j, r]) == exp, (j, r)


@pytest.mark.parametrize("shape,dtype", [
    ((2, 3, 1024, 128), torch.bfloat16), ((1, 2, 600, 3), torch.bfloat16),
    ((2, 2, 960), torch.float32), ((4096,), torch.int32), ((1, 1, 64, 5), torch.float32)])
@pytest.mark.parametrize("P", [1, 3, 8])
def test_partition_bit_exact(shape, dtype, P):
    N = shape[0] if len(shape) == 1 else shape[2]
    if N % P:
        pytest.skip("N not a multiple of P")
    g = torch.Generator().manual_seed(P)
    if dtype == torch.int32:
        x = torch.arange(N, dtype=torch.int32)
    else:
        x = torch.randn(shape, generator=g).to(dtype)
    axis = 0 if len(shape) == 1 else 2
    for layout in (W.CONTIGUOUS, W.STRIPED):
        y = ops.partition(x.cuda(), P, layout)
        z = ops.partition(y, P, layout, inverse=True)
        torch.cuda.synchronize()
        ref = OP.partition(x.view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy(), P,
                           LAYOUT[layout], axis=axis)
        got = y.cpu().view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy()
        assert np.array_equal(got, ref)
        assert torch.equal(z.cpu(), x)
    if dtype == torch.int32:     # striped position ids
        y = ops.partition(x.cuda(), P, W.STRIPED).cpu().numpy()
        assert np.array_equal(y, OP.slot_to_token(N, P, OP.STRIPED))


@pytest.mark.parametrize("alias", [False, True])
def test_lse_merge(alias):
    g = torch.Generator().manual_seed(5)
    rows, d = 3000, 128
    oa = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    ob = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    la = torch.randn(rows, generator=g) * 4
    lb = torch.randn(rows, generator=g) * 4
    la[:10] = float("-inf")
    lb[5:15] = float("-inf")
    o_ref, l_ref = OM.lse_merge(oa.double().numpy(), la.double().numpy(), ob.double().numpy(),
                                lb.double().numpy())
    doa, dla = oa.cuda(), la.cuda()
    if alias:
        o, l = ops.lse_merge(doa, dla, ob.cuda(), lb.cuda(), out=doa, lse_out=dla)
    else:
        o, l = ops.lse_merge(doa, dla, ob.cuda(), lb.cuda())
    torch.cuda.synchronize()
    o, l = o.float().cpu().numpy(), l.cpu().numpy()
    assert np.abs(o - o_ref).max() <= O_MAX
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.abs(l[fin] - l_ref[fin]).max() <= LSE_MAX
    assert np.all(o[5:10] == 0)


def test_lse_merge_of_split_keys_equals_full_attention():
    """The same queries attended on the GPU to two key halves separately and
    merged equal the attention over all keys (denominator split of the
    1cademy page)."""
    w = W.Workload("split", 1, 2, 1024, 128, 1, W.CONTIGUOUS, False, 9)
    q, k, v = W.make_qkv(w)
    half = 512
    qh = q[:, :, :half].contiguous()
    dq = qh.cuda()
    parts = []
    for sl in (slice(0, half), slice(half, 1024)):
        dk = k[:, :, sl].contiguous().cuda()
        dv = v[:, :, sl].contiguous().cuda()
        parts.append(ops.attn_fwd(dq, dk, dv, 1, W.CONTIGUOUS, False))
    (oa, la), (ob, lb) = parts
    om, lm = ops.lse_merge(oa, la, ob, lb)
    torch.cuda.synchronize()
    o_ref = np.empty((1, 2, half, 128))
    lse_ref = np.empty((1, 2, half))
    for h in range(2):
        o_ref[0, h], lse_ref[0, h] = OA.attention(qh[0, h].double().numpy(),
                                                  k[0, h].double().numpy(),
                                                  v[0, h].double().numpy(), w.scale, False)
    assert_close(om.float().cpu().numpy(), lm.cpu().numpy(), o_ref, lse_ref, "merged halves")


@pytest.mark.parametrize("layout", [W.STRIPED, W.CONTIGUOUS])
def test_o_f32_output_rounds_to_the_bf16_output(layout):
    """RA_O_F32 writes the same O before its final rounding: rounding it to
    bf16 (nearest even) gives the bf16 output bit for bit, lse identical, and
    it is at least as close to the oracle."""
    w = W.Workload("of32", 1, 2, 2048, 128, 4, layout, True, 13, qk_scale_up=3.0)
    q, k, v = W.make_qkv(w)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o16, l16 = ops.attn_fwd(dq, dk, dv, w.P, layout, True)
    o32, l32 = ops.attn_fwd(dq, dk, dv, w.P, layout, True, o_f32=True)
    torch.cuda.synchronize()
    assert o32.dtype == torch.float32
    assert torch.equal(o32.to(torch.bfloat16), o16)
    assert torch.equal(l32, l16)
    perm = OP.slot_to_token(w.N, w.P, LAYOUT[layout])
    o_ref, _ = oracle_full(q, k, v, True, w.scale)
    e32 = np.abs(o32.cpu().numpy()[:, :, np.argsort(perm)] - o_ref).mean()
    e16 = np.abs(o16.float().cpu().numpy()[:, :, np.argsort(perm)] - o_ref).mean()
    assert e32 <= e16


TOKEN_CASES = [
    # (B, H, N, d, P, layout, causal)
    (1, 2, 2048, 128, 4, W.STRIPED, True),
    (2, 3, 600, 128, 3, W.STRIPED, True),        # c = 200: ragged tiles
    (1, 2, 1500, 64, 5, W.STRIPED, False),
    (1, 2, 1024, 128, 4, W.CONTIGUOUS, True),
    (1, 2, 4096, 128, 4, W.ZIGZAG, True),
    (1, 1, 262144, 128, 16, W.STRIPED, True),    # stress shape, one head
]


@pytest.mark.parametrize("case", TOKEN_CASES, ids=lambda c: "B{}H{}N{}d{}P{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "csz"[c[5]], "C" if c[6] else "F"))
def test_token_order_is_bit_identical_to_partitioned_path(case):
    """RA_TOKEN_ORDER (the stripe applied in the TMA addressing and the
    epilogue) gives exactly the partition / attention / inverse-partition
    result."""
    B, H, N, d, P, layout, causal = case
    w = W.Workload("tok", B, H, N, d, P, layout, causal, seed=N + P, qk_scale_up=3.0)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    o_t, l_t = ops.attn_fwd(q, k, v, P, layout, causal, token_order=True)
    if layout == W.CONTIGUOUS:
        o_r, l_r = ops.attn_fwd(q, k, v, P, layout, causal)
    else:
        qp, kp, vp = (ops.partition(t, P, layout) for t in (q, k, v))
        o_p, l_p = ops.attn_fwd(qp, kp, vp, P, layout, causal)
        o_r = ops.partition(o_p, P, layout, inverse=True)
        l_r = ops.partition(l_p, P, layout, inverse=True)
    o32, _ = ops.attn_fwd(q, k, v, P, layout, causal, token_order=True, o_f32=True)
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    assert torch.equal(o_t, o_r)
    assert torch.equal(l_t, l_r)
    assert torch.equal(o32.to(torch.bfloat16), o_t)


@pytest.mark.parametrize("o_f32", [False, True])
def test_output_alignment_16_and_32_bytes_give_identical_results(o_f32):
    """O rows are written with 32-byte stores when the output is 32-byte
    aligned and with 16-byte stores otherwise (the ABI asks 16); both paths
    give the same bits."""
    w = W.Workload("align", 1, 2, 2048, 128, 4, W.STRIPED, True, 19, qk_scale_up=3.0)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    dt = torch.float32 if o_f32 else torch.bfloat16
    esz = 4 if o_f32 else 2
    n = q.numel()
    big = torch.empty(n + 32 // esz, dtype=dt, device="cuda")
    o_32 = big[:n].view(q.shape)
    o_16 = big[16 // esz:16 // esz + n].view(q.shape)
    assert o_32.data_ptr() % 32 == 0 and o_16.data_ptr() % 32 == 16
    o1, l1 = ops.attn_fwd(q, k, v, w.P, w.layout, True, out=o_32, o_f32=o_f32)
    r1, rl1 = o1.clone(), l1.clone()
    o2, l2 = ops.attn_fwd(q, k, v, w.P, w.layout, True, out=o_16, o_f32=o_f32)
    torch.cuda.synchronize()
    assert ops.device_fault() == 0
    assert torch.equal(r1, o2) and torch.equal(rl1, l2)
