"""Where the forward kernel's cycles go: per-phase clock64 counts of the
softmax warps and the MMA warp, per tile, from the profiling build.

    python -m long_context_exact_attn_b200.phase_profile [--workload NAME] [--heads H]

Builds libringattn_prof.so if needed (the library with RA_PROFILE=1), runs
the attention of one workload a few times, reads the counters through
ra_fwd_phase_profile and prints the average cycles per tile of each phase
(softmax: per warp and tile it computes; MMA: per key-tile step).  The
timers cost a few per cent; the numbers describe the kernel, not its speed.
"""

import argparse
import json

import torch

from . import build, ops
from . import workloads as W

# The first part of P is keys 0-63, or 0-95 in the work-list instance
# (small striped problems).
SOFTMAX_PHASES = ["loop, skips, epilogue", "wait for S", "load S", "row max and decision",
                  "exps of P's first part, O rescale, publish", "exps of the rest, publish"]
MMA_PHASES = ["issue", "wait next K", "wait V", "wait P (first part)", "wait P (rest)",
              "wait released O"]


def summarize(counters):
    """Cycles per tile, averaged over the CTAs that ran: softmax warps (slots
    0-7) and the MMA warp (slot 8)."""
    soft = [0] * 8
    mma = [0] * 8
    for cta in counters:
        for slot in range(8):
            for k in range(8):
                soft[k] += cta[slot][k]
        for k in range(8):
            mma[k] += cta[8][k]
    out = {}
    if soft[7]:
        out["softmax_cycles_per_tile"] = {n: soft[i] / soft[7] for i, n in enumerate(SOFTMAX_PHASES)}
        out["softmax_tiles"] = soft[7]
    if mma[7]:
        out["mma_cycles_per_step"] = {n: mma[i] / mma[7] for i, n in enumerate(MMA_PHASES)}
        out["mma_steps"] = mma[7]
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=W.STRESS_256K.name, choices=list(W.BY_NAME))
    ap.add_argument("--heads", type=int, default=0, help="override the head count")
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args()
    ops.use_library(build.build(profile=True, quiet=True))
    w = W.BY_NAME[a.workload]
    if a.heads:
        w = w.with_(H=a.heads)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    if w.layout != W.CONTIGUOUS:
        q, k, v = (ops.partition(t, w.P, w.layout) for t in (q, k, v))
    ops.attn_fwd(q, k, v, w.P, w.layout, w.causal)      # warm-up
    torch.cuda.synchronize()
    ops.fwd_phase_profile()                             # clear
    for _ in range(a.launches):
        ops.attn_fwd(q, k, v, w.P, w.layout, w.causal)
    torch.cuda.synchronize()
    if ops.device_fault():
        raise RuntimeError("device fault during the profiled launches")
    res = summarize(ops.fwd_phase_profile())
    res["workload"] = w.name if not a.heads else f"{w.name} (H={w.H})"
    res["launches"] = a.launches
    print(json.dumps(res, indent=1))


if __name__ == "__main__":
    main()
