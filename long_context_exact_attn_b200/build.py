"""Build libringattn.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m long_context_exact_attn_b200.build [--verbose-ptxas] [--profile]

The shared library lands next to this file and is what ``ops`` loads.
``--profile`` builds libringattn_prof.so instead: the same library with the
forward kernel's phase counters compiled in (RA_PROFILE=1, read through
ra_fwd_phase_profile; see ``phase_profile``).
CUDA runtime is linked statically; the driver entry point for tensor maps is
looked up at run time, so only libcuda (the driver) is needed to run it.
"""

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libringattn.so")
PROF_LIB = os.path.join(HERE, "libringattn_prof.so")
SOURCES = ["api.cu", "attn_fwd.cu", "attn_bwd.cu", "aux_kernels.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(HERE, "..", "include", "ringattn.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force=False, verbose_ptxas=False, quiet=False, profile=False):
    lib = PROF_LIB if profile else LIB
    if not force and not verbose_ptxas and not _stale(lib):
        return lib
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-cudart", "static", "--expt-relaxed-constexpr",
           "-I", os.path.join(HERE, "..", "include"), "-o", lib + ".tmp"]
    if profile:
        cmd += ["-DRA_PROFILE=1"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libringattn.so")
    if verbose_ptxas or not quiet:
        out = (res.stdout + res.stderr).strip()
        if out:
            print(out)
    os.replace(lib + ".tmp", lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="build libringattn_prof.so with the forward kernel's phase counters")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, profile=a.profile))


if __name__ == "__main__":
    main()
