"""The Python binding refuses, before any launch, caller-provided outputs that
do not match what the library will write, and tensors on the wrong device;
the C library never sees such a call (no kernel runs, the device fault word
stays clear)."""

import pytest
import torch

from long_context_exact_attn_b200 import ops

pytestmark = pytest.mark.gpu

B, H, N, D, P = 1, 2, 512, 64, 4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    assert ops.device_fault() == 0
    yield
    torch.cuda.synchronize()
    assert ops.device_fault() == 0


def qkv():
    g = torch.Generator(device="cuda").manual_seed(5)
    return [torch.randn(B, H, N, D, device="cuda", generator=g).to(torch.bfloat16)
            for _ in range(3)]


def bf16(*shape):
    return torch.empty(*shape, dtype=torch.bfloat16, device="cuda")


def f32(*shape):
    return torch.empty(*shape, dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("kw", [
    dict(out=lambda: bf16(B, H, N // 2, D)),                 # too short
    dict(out=lambda: f32(B, H, N, D)),                       # float32 without o_f32
    dict(out=lambda: bf16(B, H, N, 2 * D)[..., :D]),         # not contiguous
    dict(out=lambda: torch.empty(B, H, N, D, dtype=torch.bfloat16)),   # host memory
    dict(lse=lambda: f32(B, H, N - 1)),
    dict(lse=lambda: bf16(B, H, N)),
])
def test_attn_fwd_refuses_mismatched_outputs(kw):
    q, k, v = qkv()
    args = {n: f() for n, f in kw.items()}
    with pytest.raises(ValueError):
        ops.attn_fwd(q, k, v, P, ops.STRIPED, **args)


def test_attn_fwd_o_f32_output_must_be_float32():
    q, k, v = qkv()
    with pytest.raises(ValueError):
        ops.attn_fwd(q, k, v, P, ops.STRIPED, o_f32=True, out=bf16(B, H, N, D))
    o, _ = ops.attn_fwd(q, k, v, P, ops.STRIPED, o_f32=True, out=f32(B, H, N, D))
    assert o.dtype == torch.float32


def test_attn_bwd_refuses_mismatched_outputs():
    q, k, v = qkv()
    o, lse = ops.attn_fwd(q, k, v, P, ops.STRIPED)
    do = torch.randn_like(o)
    for kw in (dict(dq=bf16(B, H, N // 2, D)), dict(dk=f32(B, H, N, D)),
               dict(dv=bf16(B, H, N, 2 * D)[..., :D]), dict(workspace=f32(B * H * N - 1))):
        with pytest.raises(ValueError):
            ops.attn_bwd(q, k, v, o, do, lse, P, ops.STRIPED, **kw)
    with pytest.raises(ValueError):
        ops.attn_bwd(q, k, v, o, do, lse[..., :-1].contiguous(), P, ops.STRIPED)


def test_other_entries_refuse_mismatched_outputs():
    q, k, v = qkv()
    with pytest.raises(ValueError):
        ops.partition(q, P, ops.STRIPED, out=bf16(B, H, N, D // 2))
    with pytest.raises(ValueError):
        ops.partition_rope(q, P, ops.STRIPED, out=f32(B, H, N, D))
    c = N // P
    qs, ks, vs = (t[:, :, :c].contiguous() for t in (q, k, v))
    with pytest.raises(ValueError):
        ops.attn_fwd_block(qs, ks, vs, 1, 0, P, ops.STRIPED, lse=f32(B, H, c + 1))
    o, lse = ops.attn_fwd_block(qs, ks, vs, 1, 0, P, ops.STRIPED)
    acc, lacc = f32(B, H, c, D), f32(B, H, c)
    with pytest.raises(ValueError):
        ops.lse_merge_acc(acc, lacc, o, lse, first=True, final_out=bf16(B, H, c - 1, D))
    with pytest.raises(ValueError):
        ops.lse_merge(o, lse, o, lse, out=bf16(B, H, c, D + 8))
    with pytest.raises(ValueError):
        ops.lse_merge(o, lse, o, lse, lse_out=f32(B, H, c, 1))
    ws = torch.empty(ops.attn_fwd_host_workspace_bytes(N, D, ops.STRIPED, 1), dtype=torch.uint8,
                     device="cuda")
    qh, kh, vh = (t.cpu() for t in (q, k, v))
    with pytest.raises(ValueError):
        ops.attn_fwd_host(qh, kh, vh, P, ops.STRIPED, workspace=ws,
                          out=torch.empty(B, H, N // 2, D, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        ops.attn_fwd_host(qh, kh, vh, P, ops.STRIPED, workspace=ws, lse=f32(B, H, N))


def test_inputs_on_different_devices_are_refused():
    q, k, v = qkv()
    with pytest.raises(ValueError):
        ops.attn_fwd(q, k.cpu(), v, P, ops.STRIPED)
    if torch.cuda.device_count() > 1:
        with pytest.raises(ValueError):
            ops.attn_fwd(q, k.to("cuda:1"), v, P, ops.STRIPED)
