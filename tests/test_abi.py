"""The C ABI on the host (no GPU needed): the library loads, exports every
symbol the header declares, and refuses invalid arguments before touching
the device."""

import ctypes
import os
import re

import pytest

from long_context_exact_attn_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ringattn.h")


@pytest.fixture(scope="module")
def L():
    build.build(quiet=True)
    return ops.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("ra_partition", "ra_attn_fwd", "ra_lse_merge", "ra_status_string",
              "ra_tile_census", "ra_device_fault", "ra_version", "ra_wait_selftest",
              "ra_attn_bwd"):
        assert s in syms


def test_library_exports_every_declared_symbol(L):
    for s in declared_symbols():
        assert hasattr(L, s), s


def test_status_strings(L):
    assert ops.status_string(0) == "ok"
    for code in range(1, 16):
        assert ops.status_string(code) not in ("", "unknown status")
    assert ops.status_string(999) == "unknown status"
    assert L.ra_version() >= 100


# Fake, never-dereferenced device addresses: every call below must be refused
# by host validation before any CUDA call.
A = 1 << 40
Bp = 2 << 40
Cp = 3 << 40
Op = 4 << 40
Lp = 5 << 40
vp = ctypes.c_void_p


def attn(L, q=A, k=Bp, v=Cp, o=Op, lse=Lp, B=1, H=2, N=1024, d=128, P=4, layout=0, causal=1,
         scale=0.088):
    return L.ra_attn_fwd(vp(q), vp(k), vp(v), vp(o), vp(lse), B, H, N, d, P, layout, causal,
                         scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), 1), (dict(lse=0), 1),
    (dict(q=A + 8), 2), (dict(o=Op + 2), 2), (dict(lse=Lp + 4), 2),
    (dict(N=1000, P=3), 3), (dict(P=0), 3), (dict(N=0), 3), (dict(B=0), 3),
    (dict(d=96), 4), (dict(d=256), 4),
    (dict(layout=3), 5), (dict(layout=0x1000), 5), (dict(layout=0x1201), 5),
    (dict(scale=0.0), 6), (dict(scale=float("inf")), 6), (dict(scale=float("nan")), 6),
    (dict(scale=-1.0), 6),
    (dict(o=A), 8), (dict(lse=Op + 64), 8),
])
def test_attn_fwd_rejects_invalid_arguments(L, kw, code):
    assert attn(L, **kw) == code


@pytest.mark.parametrize("kw,limit,code", [
    (dict(q=0), 1_000_000, 1), (dict(d=96), 1_000_000, 4), (dict(layout=3), 1_000_000, 5),
    (dict(), 10, 3), (dict(), 20_000_000_000, 3),
])
def test_abort_selftest_validates_like_attn_fwd(L, kw, limit, code):
    a = dict(q=A, k=Bp, v=Cp, o=Op, lse=Lp, B=1, H=2, N=1024, d=128, P=4, layout=0, causal=1,
             scale=0.088)
    a.update(kw)
    assert L.ra_attn_abort_selftest(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["o"]), vp(a["lse"]),
                                    a["B"], a["H"], a["N"], a["d"], a["P"], a["layout"],
                                    a["causal"], a["scale"], limit, None) == code


def test_partition_rejects_invalid_arguments(L):
    P = L.ra_partition
    assert P(None, vp(Bp), 1, 1, 16, 4, 4, 1, 0, 0, None) == 1
    assert P(vp(A), vp(Bp), 1, 1, 16, 4, 4, 7, 0, 0, None) == 5
    assert P(vp(A), vp(Bp), 1, 1, 16, 4, 4, 1, 0, 9, None) == 7
    assert P(vp(A), vp(Bp), 1, 1, 15, 4, 4, 1, 0, 0, None) == 3
    assert P(vp(A + 2), vp(Bp), 1, 1, 16, 8, 4, 1, 0, 0, None) == 2    # 16-byte rows
    assert P(vp(A), vp(A + 64), 1, 1, 16, 8, 4, 1, 0, 0, None) == 8    # overlap


def test_lse_merge_and_census_reject_invalid_arguments(L):
    M = L.ra_lse_merge
    assert M(None, vp(A), vp(Bp), vp(Cp), vp(Op), vp(Lp), 4, 8, None) == 1
    assert M(vp(A), vp(A + 1024), vp(Bp), vp(Cp), vp(Op), vp(Lp), 4, 12, None) == 3
    assert M(vp(A + 4), vp(A + 1024), vp(Bp), vp(Cp), vp(Op), vp(Lp), 4, 8, None) == 2
    assert M(vp(A), vp(Lp), vp(Bp), vp(Cp), vp(A + 16), vp(Lp + 64), 4, 8, None) == 8
    C = L.ra_tile_census
    assert C(16, 4, 0, 1, None, None) == 1
    assert C(16, 3, 0, 1, vp(A), None) == 3
    assert C(16, 4, 3, 1, vp(A), None) == 5
    assert L.ra_device_fault(None) == 1
    assert L.ra_wait_selftest(10, None) == 3
    assert L.ra_wait_selftest(2 * 10**10, None) == 3


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()


def bwd(L, q=A, k=Bp, v=Cp, o=Op, do=6 << 40, lse=Lp, dq=7 << 40, dk=8 << 40, dv=9 << 40,
        ws=10 << 40, B=1, H=2, N=1024, d=128, P=4, layout=1, causal=1, scale=0.088):
    return L.ra_attn_bwd(vp(q), vp(k), vp(v), vp(o), vp(do), vp(lse), vp(dq), vp(dk), vp(dv),
                         vp(ws), B, H, N, d, P, layout, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ws=0), 1), (dict(do=0), 1), (dict(dq=(7 << 40) + 8), 2), (dict(ws=(10 << 40) + 4), 2),
    (dict(N=1000, P=3), 3), (dict(d=32), 4), (dict(layout=0x101), 5), (dict(layout=0x201), 5),
    (dict(scale=0.0), 6), (dict(dq=A), 8), (dict(dk=7 << 40), 8), (dict(ws=Lp), 8),
])
def test_attn_bwd_rejects_invalid_arguments(L, kw, code):
    assert bwd(L, **kw) == code


def bwd_noalloc(L, q=A, k=Bp, v=Cp, o=Op, do=6 << 40, lse=Lp, dq=7 << 40, dk=8 << 40, dv=9 << 40,
                B=1, H=2, N=1024, d=128, P=4, layout=1, causal=1, scale=0.088):
    return L.ra_attn_bwd_noalloc(vp(q), vp(k), vp(v), vp(o), vp(do), vp(lse), vp(dq), vp(dk),
                                 vp(dv), B, H, N, d, P, layout, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dv=0), 1), (dict(dq=(7 << 40) + 8), 2), (dict(N=1000, P=3), 3), (dict(d=32), 4),
    (dict(layout=0x101), 5), (dict(scale=0.0), 6), (dict(dq=A), 8), (dict(dk=7 << 40), 8),
    # one row past the built-in scratch (1048576 floats), and far past it
    (dict(B=1, H=1, N=(1 << 20) + 128, P=1), 12), (dict(B=4, H=16, N=131072, P=8), 12),
])
def test_attn_bwd_noalloc_rejects_invalid_arguments(L, kw, code):
    assert bwd_noalloc(L, **kw) == code


def prope(L, src=A, dst=Bp, B=1, H=2, N=1024, d=128, P=4, layout=1, pairing=0, base=10000.0):
    return L.ra_partition_rope(vp(src), vp(dst), B, H, N, d, P, layout, pairing, base, None)


@pytest.mark.parametrize("kw,code", [
    (dict(src=0), 1), (dict(dst=A + 16), 8), (dict(dst=Bp + 8), 2), (dict(N=1000, P=3), 3),
    (dict(d=72), 4), (dict(d=8), 4), (dict(d=1024), 4), (dict(layout=3), 5),
    (dict(pairing=2), 13), (dict(base=1.0), 13), (dict(base=float("inf")), 13),
    (dict(base=float("nan")), 13), (dict(B=0), 3),
])
def test_partition_rope_rejects_invalid_arguments(L, kw, code):
    assert prope(L, **kw) == code


def blk(L, q=A, k=Bp, v=Cp, o=Op, lse=Lp, B=1, H=2, c=256, d=128, j=1, kb=0, P=4, layout=1,
        causal=1, scale=0.088):
    return L.ra_attn_fwd_block(vp(q), vp(k), vp(v), vp(o), vp(lse), B, H, c, d, j, kb, P, layout,
                               causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(v=0), 1), (dict(o=Op + 8), 2), (dict(j=4), 3), (dict(kb=-1), 3), (dict(c=0), 3),
    (dict(d=96), 4), (dict(layout=0x101), 5), (dict(layout=0x202), 5), (dict(scale=0.0), 6),
    (dict(o=A), 8), (dict(lse=Cp + 64), 8),
    # a float32 partial (RA_O_F32) is twice as long: just below q it overlaps q
    (dict(layout=0x201, o=A - 2 * 256 * 128 * 2), 8),
])
def test_attn_fwd_block_rejects_invalid_arguments(L, kw, code):
    assert blk(L, **kw) == code


def macc(L, oa=A, la=Bp, ob=Cp, lb=Op, of=Lp, rows=256, d=128, mode=2):
    return L.ra_lse_merge_acc(vp(oa), vp(la), vp(ob), vp(lb), vp(of), rows, d, mode, None)


@pytest.mark.parametrize("kw,code", [
    (dict(oa=0), 1), (dict(of=0), 1), (dict(mode=8), 5), (dict(d=12), 3), (dict(rows=-1), 3),
    (dict(oa=A + 4), 2), (dict(ob=A + 4096), 8), (dict(of=Cp), 8),
    # a float32 partial (RA_MERGE_F32_PARTIAL) is twice as long as a bf16 one
    (dict(mode=6, of=Cp + 256 * 128 * 2), 8),
])
def test_lse_merge_acc_rejects_invalid_arguments(L, kw, code):
    assert macc(L, **kw) == code


def host(L, q=A, k=Bp, v=Cp, o=Op, lse=Lp, B=1, H=2, N=1024, d=128, P=4, layout=1, causal=1,
         scale=0.088, ws=6 << 40, wsb=1 << 30):
    return L.ra_attn_fwd_host(vp(q), vp(k), vp(v), vp(o), vp(lse), B, H, N, d, P, layout, causal,
                              scale, vp(ws), wsb, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ws=0), 1), (dict(o=0), 1), (dict(ws=(6 << 40) + 128), 2), (dict(N=1000, P=3), 3),
    (dict(d=96), 4), (dict(layout=3), 5), (dict(scale=-1.0), 6), (dict(wsb=2105343), 14),
    (dict(wsb=0), 14),
])
def test_attn_fwd_host_rejects_invalid_arguments(L, kw, code):
    assert host(L, **kw) == code


def test_host_workspace_formula(L):
    # per head and slot: q, k, v, o ([N, d] bf16) and lse ([N] float32), all
    # in token order whatever the layout; two slots
    assert L.ra_attn_fwd_host_workspace(1024, 128, 1, 1) == 2 * (4 * 262144 + 4096)
    assert L.ra_attn_fwd_host_workspace(1024, 128, 0, 3) == 2 * 3 * (4 * 262144 + 4096)
    assert L.ra_attn_fwd_host_workspace(1000, 64, 2, 1) == 2 * (4 * 128000 + 4096)
    assert L.ra_attn_fwd_host_workspace(0, 64, 1, 1) == -1


@pytest.mark.parametrize("fn,kw,code", [
    ("fwd", dict(layout=2, N=1024, P=4), 3),          # c = 256: not a multiple of 512
    ("fwd", dict(layout=2, N=2048, P=4), None),       # valid sizes: passes validation
    ("bwd", dict(layout=2), 3),                        # zigzag backward: c = 256 too short
])
def test_zigzag_validation(L, fn, kw, code):
    if fn == "fwd":
        st = attn(L, **kw)
        if code is None:
            assert st not in (3, 5)                  # fails later (no GPU here), not on sizes
        else:
            assert st == code
    else:
        assert bwd(L, **kw) == code


def test_zigzag_partition_needs_even_shards(L):
    assert L.ra_partition(vp(A), vp(Bp), 1, 1, 600, 8, 200, 2, 0, 0, None) == 3   # c = 3


def test_o_f32_flag_validation(L):
    # float32 O is twice the size: an o that overlaps q only in its second half
    tb = 2 * 1024 * 128 * 2
    assert attn(L, o=A - tb - tb // 2, layout=0x201) == 8
    assert attn(L, o=A - tb - tb // 2, layout=0x001) != 8


BIG = 1 << 33    # with two more such factors B*H*N wraps around int64


@pytest.mark.parametrize("call", [
    lambda L: attn(L, B=BIG, H=BIG, N=BIG, P=1),
    lambda L: attn(L, B=1 << 21, H=1 << 21, N=1024),
    lambda L: host(L, B=BIG, H=BIG, N=BIG, P=1),
    lambda L: bwd(L, B=BIG, H=BIG, N=BIG, P=1),
    lambda L: bwd_noalloc(L, B=BIG, H=BIG, N=BIG, P=1),
    lambda L: blk(L, B=BIG, H=BIG, c=256),
    lambda L: L.ra_partition(vp(A), vp(Bp), BIG, BIG, BIG, 8, 1, 0, 0, 0, None),
    lambda L: L.ra_partition(vp(A), vp(Bp), 1, 1, 16, 1 << 62, 4, 0, 0, 0, None),
    lambda L: prope(L, B=BIG, H=BIG, N=BIG, P=1),
    lambda L: macc(L, d=1 << 40),
])
def test_sizes_that_overflow_int64_are_refused(L, call):
    # the product of the sizes is checked factor by factor, never computed
    # past 2^62
    assert call(L) == 3


def test_host_workspace_overflow_is_refused(L):
    assert L.ra_attn_fwd_host_workspace(1 << 31, 128, 1, 1) == -1
    assert L.ra_attn_fwd_host_workspace(1024, 2048, 1, 1) == -1
    assert L.ra_attn_fwd_host_workspace(1 << 30, 128, 1, 1 << 40) == -1


C_CALLER = r"""
#include "ringattn.h"
#include <stdio.h>
int main(void) {
  if (ra_version() < 100) return 2;
  if (ra_attn_fwd(0, 0, 0, 0, 0, 1, 1, 16, 64, 4, RA_STRIPED, 1, 0.125f, 0) != RA_ERR_NULL)
    return 3;
  if (ra_attn_fwd_host_workspace(1024, 128, RA_STRIPED, 1) <= 0) return 4;
  printf("%s\n", ra_status_string(RA_ERR_SHAPE));
  return 0;
}
"""


def test_header_is_plain_c_and_links(L, tmp_path):
    # the boundary is a C ABI: the header compiles as strict C11 and a C
    # program links against the library and calls it
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(ops.LIB_PATH)
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.dirname(HEADER), str(src), "-L", libdir, "-lringattn",
                        "-Wl,-rpath," + libdir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip() == ops.status_string(3)


def test_phase_profile_needs_the_profiling_build(L):
    """The regular library keeps no phase counters: RA_ERR_NOPROFILE (15)
    without touching the device; a NULL output is refused first."""
    buf = (ctypes.c_uint64 * (160 * 10 * 8))()
    assert L.ra_fwd_phase_profile(buf, len(buf)) == 15
    assert L.ra_fwd_phase_profile(None, len(buf)) == 1
    with pytest.raises(ops.RingAttnError):
        ops.fwd_phase_profile()
