"""Python binding of libringattn.so (argument marshalling only).

Every function here validates nothing beyond what is needed to build the
call, hands raw device pointers, sizes and the current CUDA stream to the
C ABI (include/ringattn.h), and raises ``RingAttnError`` on a non-zero
status.  There is no fallback: if the library is missing or the device is
not an sm_100 GPU, calls fail loudly.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libringattn.so")

CONTIGUOUS = 0
STRIPED = 1
ZIGZAG = 2
SCHED_FREE = 0x100
O_F32 = 0x200
TOKEN_ORDER = 0x400
CTA_PAIR = 0x800

BF16 = 0
F32 = 1
I32 = 2

_DTYPE_CODE = {torch.bfloat16: BF16, torch.float32: F32, torch.int32: I32}

_lib = None


class RingAttnError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


def use_library(path):
    """Load the C library from `path` instead of the default (before the first
    call; e.g. the profiling build libringattn_prof.so)."""
    global LIB_PATH
    if _lib is not None and os.path.abspath(path) != os.path.abspath(LIB_PATH):
        raise RuntimeError("the library is already loaded from " + LIB_PATH)
    LIB_PATH = path


def lib():
    """The loaded C library (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_exact_attn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, vp, i32, f32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.ra_status_string.restype = ctypes.c_char_p
        L.ra_status_string.argtypes = [i32]
        L.ra_version.restype = i32
        L.ra_version.argtypes = []
        L.ra_partition.restype = i32
        L.ra_partition.argtypes = [vp, vp, i64, i64, i64, i64, i32, i32, i32, i32, vp]
        L.ra_attn_fwd.restype = i32
        L.ra_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, i32, f32, vp]
        L.ra_attn_bwd.restype = i32
        L.ra_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i32,
                                  i32, i32, f32, vp]
        L.ra_attn_fwd_host.restype = i32
        L.ra_attn_fwd_host.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, i32,
                                       f32, vp, i64, vp]
        L.ra_attn_fwd_host_workspace.restype = i64
        L.ra_attn_fwd_host_workspace.argtypes = [i64, i64, i32, i64]
        L.ra_attn_fwd_block.restype = i32
        L.ra_attn_fwd_block.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, i32,
                                        i32, i32, f32, vp]
        L.ra_lse_merge_acc.restype = i32
        L.ra_lse_merge_acc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, vp]
        L.ra_partition_rope.restype = i32
        L.ra_partition_rope.argtypes = [vp, vp, i64, i64, i64, i64, i32, i32, i32, f32, vp]
        L.ra_attn_bwd_noalloc.restype = i32
        L.ra_attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                          i32, i32, i32, f32, vp]
        L.ra_lse_merge.restype = i32
        L.ra_lse_merge.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, vp]
        L.ra_tile_census.restype = i32
        L.ra_tile_census.argtypes = [i64, i32, i32, i32, vp, vp]
        L.ra_wait_selftest.restype = i32
        L.ra_wait_selftest.argtypes = [i64, vp]
        L.ra_attn_abort_selftest.restype = i32
        L.ra_attn_abort_selftest.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, i32,
                                             i32, f32, i64, vp]
        L.ra_device_fault.restype = i32
        L.ra_device_fault.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.ra_fwd_phase_profile.restype = i32
        L.ra_fwd_phase_profile.argtypes = [ctypes.POINTER(ctypes.c_uint64), i64]
        _lib = L
    return _lib


def status_string(status):
    return lib().ra_status_string(int(status)).decode()


def _check(status, where):
    if status != 0:
        raise RingAttnError(status, where)


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _cuda_contig(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _like(t, name, shape, dtype, device):
    """A caller-provided output: CUDA, contiguous, of the expected shape and
    dtype, on the inputs' device (the library writes exactly that many bytes)."""
    _cuda_contig(t, name)
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} of shape {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")
    return t


def _same_device(*named):
    dev = named[0][1].device
    for n, t in named[1:]:
        if t.device != dev:
            raise ValueError(f"{n} is on {t.device}, expected {dev}")


def _launch(where, t, fn, *args):
    """One C entry point, called with t's device current (the library works on
    the current device); raises on a non-zero status."""
    with torch.cuda.device(t.device):
        _check(fn(*args), where)


def partition(x, P, layout, inverse=False, out=None):
    """Token order -> layout order (or back, ``inverse=True``) along dim -2 of
    a [B, H, N, d] tensor, or along the only dim of an [N] tensor (position
    ids).  bf16, float32 or int32."""
    _cuda_contig(x, "x")
    if x.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if x.dim() == 1:
        B, H, N, d = 1, 1, x.shape[0], 1
    elif x.dim() == 4:
        B, H, N, d = x.shape
    elif x.dim() == 3:           # [B, H, N] (e.g. lse)
        B, H, N = x.shape
        d = 1
    else:
        raise ValueError("expected [N], [B, H, N] or [B, H, N, d]")
    out = torch.empty_like(x) if out is None else _like(out, "out", x.shape, x.dtype, x.device)
    _launch("ra_partition", x, lib().ra_partition, _ptr(x), _ptr(out), B, H, N, d, int(P),
            int(layout), int(bool(inverse)), _DTYPE_CODE[x.dtype], _stream(x))
    return out


def attn_fwd(q, k, v, P, layout, causal=True, scale=None, sched_free=False, out=None, lse=None,
             o_f32=False, token_order=False, cta_pair=False):
    """Exact blockwise attention forward; q, k, v: [B, H, N, d] bf16 CUDA
    tensors in LAYOUT order (in token order with ``token_order``: the
    kernel applies the layout's permutation itself).  Returns (o [B, H, N, d]
    bf16, or float32 with ``o_f32``, lse [B, H, N] float32), in the same
    order as the inputs.  ``cta_pair`` selects the two-SM (cluster of two)
    form of the kernel where it applies (RA_CTA_PAIR: same results, slower
    on the shapes measured)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda_contig(t, n)
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{n} must be bfloat16")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, H, N, d] of the same shape")
    _same_device(("q", q), ("k", k), ("v", v))
    B, H, N, d = q.shape
    if scale is None:
        scale = d ** -0.5
    odt = torch.float32 if o_f32 else torch.bfloat16
    out = (torch.empty(q.shape, dtype=odt, device=q.device) if out is None
           else _like(out, "out", q.shape, odt, q.device))
    lse = (torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None
           else _like(lse, "lse", (B, H, N), torch.float32, q.device))
    lay = (int(layout) | (SCHED_FREE if sched_free else 0) | (O_F32 if o_f32 else 0)
           | (TOKEN_ORDER if token_order else 0) | (CTA_PAIR if cta_pair else 0))
    _launch("ra_attn_fwd", q, lib().ra_attn_fwd, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
            B, H, N, d, int(P), lay, int(bool(causal)), float(scale), _stream(q))
    return out, lse


def attn_bwd(q, k, v, o, dout, lse, P, layout, causal=True, scale=None, workspace=None,
             dq=None, dk=None, dv=None, token_order=False):
    """Gradients (dq, dk, dv) of attn_fwd; all tensors in LAYOUT order (token
    order with ``token_order``), as returned by attn_fwd on the same q, k, v.  ``workspace``: float32 with
    B*H*N elements (allocated here if not given)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _cuda_contig(t, n)
        if t.dtype != torch.bfloat16 or t.shape != q.shape:
            raise ValueError(f"{n} must be bfloat16 of q's shape")
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d]")
    B, H, N, d = q.shape
    _like(lse, "lse", (B, H, N), torch.float32, q.device)
    _same_device(("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout))
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        workspace = torch.empty(B * H * N, dtype=torch.float32, device=q.device)
    _cuda_contig(workspace, "workspace")
    if workspace.numel() < B * H * N or workspace.dtype != torch.float32 or \
            workspace.device != q.device:
        raise ValueError(f"workspace must hold B*H*N float32 on {q.device}")
    dq = torch.empty_like(q) if dq is None else _like(dq, "dq", q.shape, q.dtype, q.device)
    dk = torch.empty_like(q) if dk is None else _like(dk, "dk", q.shape, q.dtype, q.device)
    dv = torch.empty_like(q) if dv is None else _like(dv, "dv", q.shape, q.dtype, q.device)
    lay = int(layout) | (TOKEN_ORDER if token_order else 0)
    _launch("ra_attn_bwd", q, lib().ra_attn_bwd, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout),
            _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, N, d, int(P), lay,
            int(bool(causal)), float(scale), _stream(q))
    return dq, dk, dv


def attn_fwd_host_workspace_bytes(N, d, layout, heads_per_chunk):
    """Device workspace bytes ra_attn_fwd_host needs for chunks of
    ``heads_per_chunk`` heads."""
    return int(lib().ra_attn_fwd_host_workspace(N, d, int(layout), heads_per_chunk))


def attn_fwd_host(q, k, v, P, layout, causal=True, scale=None, workspace=None, out=None,
                  lse=None, sched_free=False, stream=None):
    """The whole forward from host memory: token-order host q, k, v (bf16
    [B, H, N, d], pinned for overlap) -> token-order host o, lse.  The heads
    stream through ``workspace`` (a uint8 CUDA tensor) in chunks while the
    copies of neighbouring chunks overlap the compute.  Returns (o, lse)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16 or t.shape != q.shape:
            raise ValueError(f"{n} must be a contiguous host bfloat16 tensor like q")
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d]")
    B, H, N, d = q.shape
    if scale is None:
        scale = d ** -0.5
    if workspace is None:
        raise ValueError("workspace must be a CUDA tensor")
    _cuda_contig(workspace, "workspace")
    o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, pin_memory=True) if lse is None else lse
    for n, t, shape, dt in (("out", o, q.shape, q.dtype), ("lse", lse, (B, H, N), torch.float32)):
        if t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape) or t.dtype != dt:
            raise ValueError(f"{n} must be a contiguous host {dt} tensor of shape {tuple(shape)}")
    lay = int(layout) | (SCHED_FREE if sched_free else 0)
    st = torch.cuda.current_stream(workspace.device) if stream is None else stream
    _launch("ra_attn_fwd_host", workspace, lib().ra_attn_fwd_host, _ptr(q), _ptr(k), _ptr(v),
            _ptr(o), _ptr(lse), B, H, N, d, int(P), lay, int(bool(causal)), float(scale),
            _ptr(workspace), workspace.numel() * workspace.element_size(),
            ctypes.c_void_p(st.cuda_stream))
    return o, lse


def attn_fwd_block(q, k, v, j, kb, P, layout, causal=True, scale=None, out=None, lse=None,
                   o_f32=False):
    """One round of the ring on this device: query shard j [B, H, c, d]
    against key/value block kb [B, H, c, d] (layout order), normalised over
    the block; rows that see no key of it get o = 0, lse = -inf.  With
    ``o_f32`` the partial O is float32 (rounded once, later, by the merge)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda_contig(t, n)
        if t.dtype != torch.bfloat16 or t.dim() != 4 or t.shape != q.shape:
            raise ValueError(f"{n} must be bfloat16 [B, H, c, d] like q")
    _same_device(("q", q), ("k", k), ("v", v))
    B, H, c, d = q.shape
    if scale is None:
        scale = d ** -0.5
    odt = torch.float32 if o_f32 else q.dtype
    o = (torch.empty(q.shape, dtype=odt, device=q.device) if out is None
         else _like(out, "out", q.shape, odt, q.device))
    lse = (torch.empty(B, H, c, dtype=torch.float32, device=q.device) if lse is None
           else _like(lse, "lse", (B, H, c), torch.float32, q.device))
    lay = int(layout) | (O_F32 if o_f32 else 0)
    _launch("ra_attn_fwd_block", q, lib().ra_attn_fwd_block, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
            _ptr(lse), B, H, c, d, int(j), int(kb), int(P), lay, int(bool(causal)),
            float(scale), _stream(q))
    return o, lse


MERGE_FIRST, MERGE_FINAL, MERGE_F32_PARTIAL = 1, 2, 4


def lse_merge_acc(o_acc, lse_acc, o_b, lse_b, first=False, final_out=None):
    """Fold a partial (o_b bf16 or float32, lse_b) into the float32
    accumulator (o_acc, lse_acc) in place; with ``final_out`` also write the
    merged O as bf16 there."""
    d = o_b.shape[-1]
    rows = o_b.numel() // d
    if o_acc.dtype != torch.float32 or o_acc.shape != o_b.shape or \
            o_b.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("o_acc float32 and o_b bfloat16 or float32 of the same shape")
    if lse_acc.dtype != torch.float32 or lse_b.dtype != torch.float32 or \
            lse_acc.numel() != rows or lse_b.numel() != rows:
        raise ValueError("lse_acc, lse_b: float32 with one value per row")
    for n, t in (("o_acc", o_acc), ("lse_acc", lse_acc), ("o_b", o_b), ("lse_b", lse_b)):
        _cuda_contig(t, n)
    _same_device(("o_b", o_b), ("o_acc", o_acc), ("lse_acc", lse_acc), ("lse_b", lse_b))
    mode = ((MERGE_FIRST if first else 0) | (MERGE_FINAL if final_out is not None else 0)
            | (MERGE_F32_PARTIAL if o_b.dtype == torch.float32 else 0))
    fin = None
    if final_out is not None:
        fin = _ptr(_like(final_out, "final_out", o_b.shape, torch.bfloat16, o_b.device))
    _launch("ra_lse_merge_acc", o_b, lib().ra_lse_merge_acc, _ptr(o_acc), _ptr(lse_acc),
            _ptr(o_b), _ptr(lse_b), fin, rows, d, mode, _stream(o_b))
    return o_acc, lse_acc


ROPE_INTERLEAVED, ROPE_HALF = 0, 1


def partition_rope(x, P, layout, base=10000.0, pairing=ROPE_INTERLEAVED, out=None):
    """Token order -> layout order of q or k [B, H, N, d] (bf16) with rotary
    position embedding applied at the original token positions."""
    _cuda_contig(x, "x")
    if x.dim() != 4 or x.dtype != torch.bfloat16:
        raise ValueError("x must be bfloat16 [B, H, N, d]")
    B, H, N, d = x.shape
    out = torch.empty_like(x) if out is None else _like(out, "out", x.shape, x.dtype, x.device)
    _launch("ra_partition_rope", x, lib().ra_partition_rope, _ptr(x), _ptr(out), B, H, N, d,
            int(P), int(layout), int(pairing), float(base), _stream(x))
    return out


def attn_bwd_noalloc(q, k, v, o, dout, lse, P, layout, causal, scale, dq, dk, dv):
    """attn_bwd through ra_attn_bwd_noalloc: for callers that own all device
    memory and cannot let the library (or this binding) allocate.  The outputs
    dq, dk, dv must be passed in; the scratch is the library's fixed array
    (B*H*N <= 1048576).  Calls overlapping on the GPU race on that array."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout),
                 ("dq", dq), ("dk", dk), ("dv", dv)):
        _cuda_contig(t, n)
        if t.dtype != torch.bfloat16 or t.shape != q.shape:
            raise ValueError(f"{n} must be bfloat16 of q's shape")
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d]")
    B, H, N, d = q.shape
    _like(lse, "lse", (B, H, N), torch.float32, q.device)
    _same_device(("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk),
                 ("dv", dv))
    _launch("ra_attn_bwd_noalloc", q, lib().ra_attn_bwd_noalloc, _ptr(q), _ptr(k), _ptr(v),
            _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, int(P),
            int(layout), int(bool(causal)), float(scale), _stream(q))
    return dq, dk, dv


def lse_merge(o_a, lse_a, o_b, lse_b, out=None, lse_out=None):
    """Merge two partial (o, lse) results over disjoint key sets; o: [..., d]
    bf16, lse: [...] float32."""
    if o_b.shape != o_a.shape or lse_a.shape != o_a.shape[:-1] or lse_b.shape != lse_a.shape:
        raise ValueError("o_a, o_b must match and lse_* must be o's shape without the last dim")
    if o_a.dtype != torch.bfloat16 or o_b.dtype != torch.bfloat16:
        raise ValueError("o_a, o_b must be bfloat16")
    if lse_a.dtype != torch.float32 or lse_b.dtype != torch.float32:
        raise ValueError("lse_a, lse_b must be float32")
    d = o_a.shape[-1]
    rows = o_a.numel() // d
    for n, t in (("o_a", o_a), ("lse_a", lse_a), ("o_b", o_b), ("lse_b", lse_b)):
        _cuda_contig(t, n)
    _same_device(("o_a", o_a), ("lse_a", lse_a), ("o_b", o_b), ("lse_b", lse_b))
    out = (torch.empty_like(o_a) if out is None
           else _like(out, "out", o_a.shape, torch.bfloat16, o_a.device))
    lse_out = (torch.empty_like(lse_a) if lse_out is None
               else _like(lse_out, "lse_out", lse_a.shape, torch.float32, o_a.device))
    _launch("ra_lse_merge", o_a, lib().ra_lse_merge, _ptr(o_a), _ptr(lse_a), _ptr(o_b),
            _ptr(lse_b), _ptr(out), _ptr(lse_out), rows, d, _stream(o_a))
    return out, lse_out


def tile_census(N, P, layout, causal, device="cuda"):
    """int64 [P, P, 4]: per (query shard j, round r): skipped / full /
    masked tiles and visible pairs, from the attention kernel's classifier."""
    out = torch.empty((P, P, 4), dtype=torch.int64, device=device)
    _launch("ra_tile_census", out, lib().ra_tile_census, int(N), int(P), int(layout),
            int(bool(causal)), _ptr(out), _stream(out))
    return out


def wait_selftest(limit_ns=100_000_000, device="cuda"):
    """Launch the bounded-wait self-test (a wait that nothing completes)."""
    dev = torch.device(device)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    with torch.cuda.device(dev):
        _check(lib().ra_wait_selftest(int(limit_ns), stream), "ra_wait_selftest")


def attn_abort_selftest(q, k, v, P, layout, causal=True, limit_ns=1_000_000, out=None,
                        lse=None):
    """Launch the attention kernel with its first S-ready signal withheld in
    every CTA: the main-loop waits give up after ``limit_ns``, the kernel
    drains and returns with fault code 1 (read it with ``device_fault``).
    Same arguments as attn_fwd (layout order)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda_contig(t, n)
        if t.dtype != torch.bfloat16 or t.shape != q.shape or t.dim() != 4:
            raise ValueError(f"{n} must be bfloat16 [B, H, N, d] like q")
    B, H, N, d = q.shape
    out = torch.empty_like(q) if out is None else _like(out, "out", q.shape, q.dtype, q.device)
    lse = (torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None
           else _like(lse, "lse", (B, H, N), torch.float32, q.device))
    _launch("ra_attn_abort_selftest", q, lib().ra_attn_abort_selftest, _ptr(q), _ptr(k), _ptr(v),
            _ptr(out), _ptr(lse), B, H, N, d, int(P), int(layout), int(bool(causal)),
            float(d ** -0.5), int(limit_ns), _stream(q))
    return out, lse


PROFILE_SHAPE = (160, 10, 8)   # CTAs, role slots, phases (see ra_fwd_phase_profile)


def fwd_phase_profile():
    """Read and clear the forward kernel's phase counters (profiling build
    only; the regular library raises RingAttnError with RA_ERR_NOPROFILE).
    Returns a nested list [cta][slot][phase] of cycle counts (phase 7: tiles)."""
    n = PROFILE_SHAPE[0] * PROFILE_SHAPE[1] * PROFILE_SHAPE[2]
    buf = (ctypes.c_uint64 * n)()
    _check(lib().ra_fwd_phase_profile(buf, n), "ra_fwd_phase_profile")
    c, sl, ph = PROFILE_SHAPE
    return [[[int(buf[(i * sl + j) * ph + k]) for k in range(ph)] for j in range(sl)]
            for i in range(c)]


def device_fault():
    """Read and clear the device fault word (synchronises the device)."""
    code = ctypes.c_int(0)
    st = lib().ra_device_fault(ctypes.byref(code))
    if st not in (0, 11):
        raise RingAttnError(st, "ra_device_fault")
    return code.value
