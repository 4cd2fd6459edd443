"""Benchmark: causal ring/striped attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-compare] [--no-cpu-baseline]

One step is the whole hot path over one batch of synthetic input: partition
Q, K, V into the layout order, the attention forward (all rounds of all
virtual shards), and un-partition O and lse back to token order.

Metric: useful causal attention TFLOP/s (4*d FLOPs per unmasked query-key
pair, all heads), with tokens/s and the fraction of the measured dense-BF16
tensor peak alongside.  The default workload is the stress configuration
(B=1, H=16, N=262144, d=128, P=16 striped, q/k scaled x3).  Inputs (3 GiB)
are far larger than L2 (126 MB), so no L2 flush is needed between steps.

With --gpus N > 1 (launched under torchrun) every rank runs its own replica
of the workload: the work has no exchange step on one GPU, so scaling is
weak and value = all ranks' useful FLOPs / slowest rank's time.

--impl reference times the CPU oracle (fp64 NumPy, plain definition) on a
bounded row sample of the same workload, on this machine's host cores.
"""

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_exact_attn_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0
METRIC = "causal attn fwd useful TFLOP/s & % BF16 tensor peak; tokens/s (1×B200)"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The sources the forward kernel is compiled from (its file and what it
# includes): a recorded ncu traffic figure is valid while their code (not
# their comments) is unchanged.
FWD_SOURCES = ("attn_fwd.cu", "exp2_poly.h", "ra_internal.h", "ra_ptx.cuh", "ra_tiles.cuh")


def _strip_comments(text):
    """C/C++ source without comments and blank-space runs (comment edits do
    not change the compiled kernel, so they must not invalidate a record)."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_exact_attn_b200", "csrc")
    for name in FWD_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel sources for this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload_name)
    if not e or e.get("kernel_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: clocks unknown
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.1)

    def start(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------- CPU oracle
def oracle_head(w, h):
    q, k, v = W.make_qkv_head(w, 0, h)
    return h, q.double().numpy(), k.double().numpy(), v.double().numpy()


def structured_rows(w):
    """Token indices of rows whose handling differs in the kernel: row 0 and
    the last row, every shard's first and last local row, and the rows on
    both sides of shard 0's first tile edges (layout terms)."""
    from oracle import partition as OP

    lay = {W.CONTIGUOUS: OP.CONTIGUOUS, W.STRIPED: OP.STRIPED, W.ZIGZAG: OP.ZIGZAG}[w.layout]
    slots = {0, w.N - 1}
    for j in range(w.P):
        slots.update({j * w.c, j * w.c + w.c - 1})
    for x in (127, 128, 255, 256):
        if x < w.c:
            slots.add(x)
    return sorted({OP.token_of(s // w.c, s % w.c, w.N, w.P, lay) for s in slots})


def cpu_oracle_leg(w, budget_s, seed=0, head=None):
    """Run the oracle's plain definition row by row on a bounded sample of
    the workload: the structured rows first, then uniformly random rows until
    the time budget is spent.  Returns (useful TFLOP/s, description, threads,
    (head, rows, o, lse)) -- the oracle's rows are kept so the caller can
    compare the GPU's output with them."""
    from threadpoolctl import threadpool_info

    from oracle import attention as OA

    rng = np.random.default_rng(seed)
    h, qn, kn, vn = head if head is not None else oracle_head(w, int(rng.integers(0, w.H)))
    first = structured_rows(w)
    rest = rng.permutation(w.N)[:4096]
    order = first + [int(i) for i in rest if int(i) not in set(first)]
    rows, os_, ls_ = [], [], []
    flops = 0
    t0 = time.perf_counter()
    for i in order[:4096]:
        o, lse = OA.attention_rows(qn, kn, vn, w.scale, w.causal, [int(i)])
        rows.append(int(i))
        os_.append(o[0])
        ls_.append(lse[0])
        flops += 4 * w.d * ((int(i) + 1) if w.causal else w.N)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    desc = (f"{len(rows)} query rows of head {h} of {w.name} ({len(first)} structured: row 0, "
            f"shard edges, tile edges; the rest uniform random), each against all its visible "
            f"keys; fp64 NumPy oracle; {dt:.1f} s")
    return flops / dt / 1e12, desc, threads, (h, rows, np.array(os_), np.array(ls_))


O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


def parity_of(o_gpu, lse_gpu, v0, ref):
    """Element-wise errors of the GPU's O and lse (token order, [B, H, N, d]
    and [B, H, N]) against the oracle rows of one head."""
    h, rows, o_ref, lse_ref = ref
    idx = torch.tensor(rows, dtype=torch.long, device=o_gpu.device)
    o = o_gpu[0, h].index_select(0, idx).double().cpu().numpy()
    lse = lse_gpu[0, h].index_select(0, idx).double().cpu().numpy()
    err = np.abs(o - o_ref)
    lerr = np.abs(lse - lse_ref)
    row0 = None
    if 0 in rows and v0 is not None:
        row0 = bool(np.array_equal(o[rows.index(0)], v0))
    return {"head": h, "rows": len(rows), "o_max_abs": float(err.max()),
            "o_mean_abs": float(err.mean()), "lse_max_abs": float(lerr.max()),
            "tolerance": {"o_max_abs": O_MAX, "o_mean_abs": O_MEAN, "lse_max_abs": LSE_MAX},
            "within": bool(err.max() <= O_MAX and err.mean() <= O_MEAN and lerr.max() <= LSE_MAX),
            "row0_equals_v0": row0,
            "reference": "fp64 oracle, plain definition, same bf16 inputs"}


def config_of(w, sched, world):
    """The line's config object (shared by both arms, so the two lines name
    the same workload the same way)."""
    in_bytes = 3 * w.B * w.H * w.N * w.d * 2
    if in_bytes < 4 * L2_BYTES:
        l2 = (f"inputs ({in_bytes / 2 ** 20:.0f} MiB) not much larger than L2: a "
              f"{2 * L2_BYTES / 2 ** 20:.0f} MiB buffer is written before every timed step, "
              f"outside the timed window")
    else:
        l2 = f"inputs ({in_bytes / 2 ** 30:.1f} GiB) larger than L2; no flush"
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "P": w.P,
            "layout": w.layout_name, "causal": w.causal, "schedule": sched,
            "step": "partition q,k,v -> attention -> unpartition o,lse", "l2": l2,
            "parallelism": f"replicas x{world}"}


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    vals = []
    desc = threads = None
    head = oracle_head(w, w.H - 1)
    for i in range(args.warmup + args.steps):
        rate, desc, threads, _ = cpu_oracle_leg(w, args.ref_budget, seed=i, head=head)
        if i >= args.warmup:
            vals.append(rate)
    val = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": w.useful_flops() / (val * 1e12) * 1e3,
        "ms_per_step_kind": "extrapolated_from_rows",
        "ms_per_step_note": "each step runs a bounded row sample of the workload; ms_per_step is "
                            "the whole workload's useful work at the measured row rate",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.sched, world),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU path
class Path:
    """Device buffers and the step of the hot path for one workload."""

    def __init__(self, ops, w, q, k, v, sched_free=False, layout=None):
        self.ops, self.w = ops, w
        self.layout = w.layout if layout is None else layout
        self.sched_free = sched_free
        dev = torch.device("cuda", torch.cuda.current_device())
        self.q, self.k, self.v = (t.to(dev) for t in (q, k, v))
        self.qp, self.kp, self.vp = (torch.empty_like(t) for t in (self.q, self.k, self.v))
        self.op = torch.empty_like(self.q)
        self.o = torch.empty_like(self.q)
        self.lsep = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        self.lse = torch.empty_like(self.lsep)
        self.ev_attn = []
        self.launches_per_step = 1 if self.layout == W.CONTIGUOUS else 6

    def step(self, time_attn=False):
        ops, w, P, lay = self.ops, self.w, self.w.P, self.layout
        if lay != W.CONTIGUOUS:
            for src, dst in ((self.q, self.qp), (self.k, self.kp), (self.v, self.vp)):
                ops.partition(src, P, lay, out=dst)
            qq, kk, vv = self.qp, self.kp, self.vp
        else:
            qq, kk, vv = self.q, self.k, self.v
        if time_attn:
            s = torch.cuda.current_stream()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
        ops.attn_fwd(qq, kk, vv, P, lay, w.causal, sched_free=self.sched_free,
                     out=self.o if lay == W.CONTIGUOUS else self.op,
                     lse=self.lse if lay == W.CONTIGUOUS else self.lsep)
        if time_attn:
            e1.record(s)
            self.ev_attn.append((e0, e1))
        if lay != W.CONTIGUOUS:
            ops.partition(self.op, P, lay, inverse=True, out=self.o)
            ops.partition(self.lsep, P, lay, inverse=True, out=self.lse)

    def attn_ms(self):
        torch.cuda.synchronize()
        ts = [a.elapsed_time(b) for a, b in self.ev_attn]
        self.ev_attn = []
        return ts


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank number over all ranks (nccl: on the device; gloo: host)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(flops_per_rank, ms_max, world):
    """Whole-job useful TFLOP/s: every rank's work over the slowest rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


def timed(fn, steps, world, flush=None):
    """Mean device time of fn over `steps` runs, max over ranks.  With
    `flush`, L2 is overwritten before every run and each run is timed on its
    own, so the flush stays outside the timed windows."""
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
    else:
        evs = []
        for _ in range(steps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            fn()
            e1.record(s)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    barrier(world)
    return max_over_ranks(ms, world)


def workload_leg(ops, w2, sched, world, steps):
    """One of the other configurations of the method's evaluation, timed the
    same way as the headline step (partition -> attention -> un-partition,
    L2 flushed before every step when the inputs are near L2 size)."""
    q2, k2, v2 = W.make_qkv(w2)
    pth = Path(ops, w2, q2, k2, v2, sched_free=(sched == "free"))
    in_bytes = 3 * q2.numel() * q2.element_size()
    flush = None
    if in_bytes < 4 * L2_BYTES:
        flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        flush = flush_buf.zero_
    for _ in range(3):
        pth.step()
    torch.cuda.synchronize()
    ms = timed(lambda: pth.step(time_attn=True), steps, world, flush=flush)
    attn = pth.attn_ms()
    am = max_over_ranks(statistics.median(attn), world)
    fl = w2.useful_flops()
    out = {"step_ms": round(ms, 4), "attn_ms_median": round(am, 4),
           "useful_tflops_step": round(fl * world / (ms * 1e-3) / 1e12, 1),
           "useful_tflops_attn": round(fl / (am * 1e-3) / 1e12, 1),
           "tokens_per_s": w2.B * w2.N * world / (ms * 1e-3),
           "layout": w2.layout_name, "schedule": sched, "causal": w2.causal,
           "l2_flush": flush is not None, "steps": steps}
    if ops.device_fault():
        raise RuntimeError(f"device fault in workload {w2.name}")
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.STRESS_256K.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--sched", default="owner", choices=["owner", "free"])
    ap.add_argument("--no-compare", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="head chunks of the host-buffer path (copies overlap compute)")
    ap.add_argument("--no-ring-emulate", action="store_true",
                    help="skip timing every (rank, round) block of the physical ring")
    ap.add_argument("--no-rope", action="store_true",
                    help="skip timing the stripe + RoPE partition of q")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the backward pass (dQ, dK, dV) on the same workload")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other configurations of the evaluation")
    ap.add_argument("--ref-budget", type=float, default=15.0,
                    help="seconds of CPU work per reference step")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (a reduced case of the same "
                         "per-head shape, e.g. for counter captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = W.BY_NAME[args.workload]
    if args.heads is not None and args.heads != w.H:
        w = w.with_(H=args.heads, name=f"{w.name}_H{args.heads}")

    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    from long_context_exact_attn_b200 import ops

    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ops.lib()
    peaks, peaks_src = load_peaks()
    config = config_of(w, args.sched, world)

    q, k, v = W.make_qkv(w)
    path = Path(ops, w, q, k, v, sched_free=(args.sched == "free"))
    # Inputs smaller than a few L2s: overwrite L2 before every timed step.
    in_bytes = 3 * q.numel() * q.element_size()
    flush = None
    if in_bytes < 4 * L2_BYTES:
        flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        flush = flush_buf.zero_

    for _ in range(args.warmup):
        path.step()
    torch.cuda.synchronize()
    if ops.device_fault():
        raise RuntimeError("device fault during warm-up")

    sampler = ClockSampler(local)
    sampler.start()
    ms = timed(lambda: path.step(time_attn=True), args.steps, world, flush=flush)
    clocks = sampler.stop()
    attn_ts = path.attn_ms()
    if ops.device_fault():
        raise RuntimeError("device fault during the timed steps")
    attn_ms = statistics.mean(attn_ts)
    attn_ms = max_over_ranks(attn_ms, world)

    flops = w.useful_flops()
    value = job_value(flops, ms, world)
    tokens_s = w.B * w.N * world / (ms * 1e-3)
    # the timed step's output (token order), kept on the host for the
    # comparison with the oracle's rows at the end
    o_step = path.o.cpu()
    lse_step = path.lse.cpu()

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # ra_attn_fwd_host: token-order host q, k, v in, host o, lse out; the
        # heads go through a device workspace in chunks, copies of
        # neighbouring chunks overlapping the compute
        hq, hk, hv = (t.pin_memory() for t in (q, k, v))
        ho = torch.empty(path.o.shape, dtype=path.o.dtype).pin_memory()
        hl = torch.empty(path.lse.shape, dtype=path.lse.dtype).pin_memory()
        g = max(1, -(-(w.B * w.H) // args.e2e_chunks))
        wsb = ops.attn_fwd_host_workspace_bytes(w.N, w.d, path.layout, g)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")

        def e2e_step():
            ops.attn_fwd_host(hq, hk, hv, w.P, w.layout, w.causal, workspace=ws, out=ho, lse=hl,
                              sched_free=args.sched == "free")

        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(1, min(args.steps, 5))
        e2e_ms = timed(e2e_step, n_e2e, world)
        del ws
        torch.cuda.empty_cache()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
        # Its parts, each timed alone: the attention of every head chunk on
        # device-resident token-order inputs (the kernels the host path runs),
        # and plain pinned-memory copies of the step's inputs and outputs.
        parts = None
        if w.B == 1:
            fo, fl_ = torch.empty_like(path.o), torch.empty_like(path.lse)

            def chunks():
                for h0 in range(0, w.H, g):
                    h1 = min(w.H, h0 + g)
                    ops.attn_fwd(path.q[:, h0:h1], path.k[:, h0:h1], path.v[:, h0:h1], w.P,
                                 path.layout, w.causal, sched_free=args.sched == "free",
                                 out=fo[:, h0:h1], lse=fl_[:, h0:h1], token_order=True)

            chunks()
            chunk_ms = timed(chunks, n_e2e, world)
            dq_ = torch.empty_like(path.q)

            def h2d_copy():
                for t in (hq, hk, hv):
                    dq_.copy_(t, non_blocking=True)

            def d2h_copy():
                ho.copy_(fo, non_blocking=True)
                hl.copy_(fl_, non_blocking=True)

            h2d_copy()
            h2d_ms = timed(h2d_copy, 3, world)
            d2h_ms = timed(d2h_copy, 3, world)
            del fo, fl_, dq_
            torch.cuda.empty_cache()
            parts = {"chunk_kernels_ms": chunk_ms, "exposed_copy_ms": e2e_ms - chunk_ms,
                     "h2d_alone_ms": h2d_ms, "h2d_gbs": h2d / (h2d_ms * 1e-3) / 1e9,
                     "d2h_alone_ms": d2h_ms, "d2h_gbs": d2h / (d2h_ms * 1e-3) / 1e9,
                     "note": "chunk_kernels_ms: the same head chunks attended on device-resident "
                             "token-order tensors, back to back; exposed_copy_ms = e2e - that; "
                             "copies timed alone from/to pinned host memory"}
        e2e = {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "ra_attn_fwd_host (pinned host buffers)", "heads_per_chunk": g,
               "parts": parts}

    # ---- the same step with the layout's permutation applied inside the
    # attention kernel (RA_TOKEN_ORDER: one launch, token order in and out)
    fused = None
    if not args.no_compare and path.layout != W.CONTIGUOUS:
        fo, fl = torch.empty_like(path.o), torch.empty_like(path.lse)

        def fused_step():
            ops.attn_fwd(path.q, path.k, path.v, w.P, path.layout, w.causal,
                         sched_free=path.sched_free, out=fo, lse=fl, token_order=True)

        fused_step()
        fms = timed(fused_step, max(1, min(args.steps, 5)), world, flush=flush)
        fused = {"ms_per_step": fms, "useful_tflops": flops * world / (fms * 1e-3) / 1e12,
                 "launches_per_step": 1,
                 "note": "partition and un-partition folded into the kernel's TMA "
                         "coordinates and epilogue rows (bit-identical results)"}
        del fo, fl

    # ---- the layout/schedule comparison at equal shapes (attention only)
    compare = None
    if not args.no_compare:
        compare = {}
        lays = [W.STRIPED, W.CONTIGUOUS]
        if (w.N // w.P) % 512 == 0:
            lays.append(W.ZIGZAG)      # zigzag attention needs N/P a multiple of 512
        for lay in lays:
            for sched in ("owner", "free"):
                pth = path if (lay == w.layout and sched == args.sched) else None
                if pth is None:
                    pth = Path(ops, w, q, k, v, sched_free=(sched == "free"), layout=lay)
                    pth.step()
                    torch.cuda.synchronize()
                n = 3
                for _ in range(n):
                    if flush is not None:
                        flush()
                    pth.step(time_attn=True)
                t = statistics.median(pth.attn_ms())
                t = max_over_ranks(t, world)
                compare[f"{W.LAYOUT_NAMES[lay]}_{sched}"] = {
                    "attn_ms": round(t, 3), "useful_tflops": round(flops / (t * 1e-3) / 1e12, 1)}
                if pth is not path:
                    del pth
                    torch.cuda.empty_cache()
        so, co = compare["striped_owner"]["attn_ms"], compare["contiguous_owner"]["attn_ms"]
        compare["contiguous_over_striped_owner"] = round(co / so, 3)
        if ops.device_fault():
            raise RuntimeError("device fault during the layout comparison")

    # ---- backward pass: 10 d useful FLOP per visible pair (5 products)
    backward = None
    if not args.no_backward:
        lay = path.layout
        qq, kk, vv = (path.qp, path.kp, path.vp) if lay != W.CONTIGUOUS else (path.q, path.k, path.v)
        oo = path.op if lay != W.CONTIGUOUS else path.o
        ll = path.lsep if lay != W.CONTIGUOUS else path.lse
        path.step()
        dout = torch.randn(qq.shape, device=qq.device,
                           generator=torch.Generator(device=qq.device).manual_seed(1)).to(qq.dtype)
        ws = torch.empty(qq.numel() // qq.shape[-1], dtype=torch.float32, device=qq.device)
        grads = [torch.empty_like(qq) for _ in range(3)]

        def bwd_step():
            ops.attn_bwd(qq, kk, vv, oo, dout, ll, w.P, lay, w.causal, workspace=ws,
                         dq=grads[0], dk=grads[1], dv=grads[2])

        bwd_step()
        torch.cuda.synchronize()
        n_b = max(1, min(args.steps, 3))
        bms = timed(bwd_step, n_b, world, flush=flush)
        if ops.device_fault():
            raise RuntimeError("device fault during the backward pass")
        del dout, ws, grads
        torch.cuda.empty_cache()
        # useful: 10 d FLOP per visible pair (the five products of the
        # gradient); executed: 14 d (the dQ kernel recomputes S and dP)
        useful = 2.5 * flops * world / (bms * 1e-3) / 1e12
        executed = 3.5 * flops * world / (bms * 1e-3) / 1e12
        backward = {"ms": bms, "steps": n_b, "useful_tflops": useful,
                    "executed_tflops": executed,
                    "frac_executed_of_sustained_peak":
                        executed / world / float(peaks.get("bf16_tflops_sustained",
                                                           FALLBACK_PEAKS["bf16_tflops_sustained"])),
                    "kernels": "bwd_rowdot_kernel, bwd_dkdv_kernel, bwd_dq_kernel",
                    "flop_convention": "useful 10 d per visible pair (QK^T, dO V^T, dV, dK, dQ); "
                                       "executed 14 d (S and dP recomputed for dQ)"}

    # ---- the other configurations of the evaluation (same step, own inputs)
    configs = None
    if not args.no_configs:
        configs = {}
        for w2 in (W.RING_8K, W.STRIPED_8K, W.LONG_128K):
            if w2.name == w.name:
                continue
            configs[w2.name] = workload_leg(ops, w2, args.sched, world,
                                            steps=20 if w2.N <= 8192 else 5)
            torch.cuda.empty_cache()

    # ---- the physical ring, emulated on this GPU: every (rank j, round r)
    # block of ra_attn_fwd_block timed alone; on P devices round r lasts as
    # long as its slowest rank, so sum_r max_j t(j, r) predicts the ring's
    # compute time (the K/V exchange, 2 B H c d 2 bytes per rank per round,
    # overlaps it)
    ring = None
    if not args.no_ring_emulate and rank == 0 and world == 1:
        ring = {}
        c = w.N // w.P
        for lay in (W.STRIPED, W.CONTIGUOUS):
            src = (path.q, path.k, path.v)
            if lay != W.CONTIGUOUS:
                src = tuple(ops.partition(t, w.P, lay) for t in src)
            shards = [[t[:, :, j * c:(j + 1) * c].contiguous() for j in range(w.P)] for t in src]
            del src
            o_blk = torch.empty(shards[0][0].shape, dtype=torch.float32, device="cuda")
            l_blk = torch.empty(w.B, w.H, c, dtype=torch.float32, device="cuda")
            acc = torch.empty(o_blk.shape, dtype=torch.float32, device="cuda")
            lacc = torch.empty_like(l_blk)
            # first pass warms up; each block's time is the median of the
            # three passes after it (one slow launch must not set a round)
            samples = [[[] for _ in range(w.P)] for _ in range(w.P)]
            for rep in range(4):
                for j in range(w.P):
                    for r in range(w.P):
                        kb = (j - r) % w.P
                        e0 = torch.cuda.Event(enable_timing=True)
                        e1 = torch.cuda.Event(enable_timing=True)
                        e0.record()
                        ops.attn_fwd_block(shards[0][j], shards[1][kb], shards[2][kb], j, kb, w.P,
                                           lay, w.causal, out=o_blk, lse=l_blk, o_f32=True)
                        ops.lse_merge_acc(acc, lacc, o_blk, l_blk, first=(r == 0))
                        e1.record()
                        e1.synchronize()
                        if rep:
                            samples[j][r].append(e0.elapsed_time(e1))
            t = [[statistics.median(samples[j][r]) for r in range(w.P)] for j in range(w.P)]
            del shards, o_blk, l_blk, acc, lacc
            torch.cuda.empty_cache()
            round_max = [max(t[j][r] for j in range(w.P)) for r in range(w.P)]
            total = sum(round_max)
            per_rank = [sum(t[j]) for j in range(w.P)]
            xfer = 2 * w.B * w.H * c * w.d * 2
            ring[W.LAYOUT_NAMES[lay]] = {
                "predicted_ring_ms": round(total, 3),
                "useful_tflops_on_P_gpus": round(flops / (total * 1e-3) / 1e12, 1),
                "round_max_ms": [round(x, 3) for x in round_max],
                "rank_busy_ms_min_max": [round(min(per_rank), 3), round(max(per_rank), 3)],
                "kv_bytes_per_rank_per_round": xfer,
                "kv_ms_per_round_at_770GBs": round(xfer / 770e9 * 1e3, 4)}
        if ops.device_fault():
            raise RuntimeError("device fault during the ring emulation")
        ring["contiguous_over_striped"] = round(
            ring["contiguous"]["predicted_ring_ms"] / ring["striped"]["predicted_ring_ms"], 3)
        ring["note"] = ("per-round block (float32 partial) + merge kernels of every rank run "
                        "one at a time on this GPU (median of 3 timings each); P GPUs would "
                        "run each round's ranks concurrently")

    # ---- stripe + RoPE of q and k (memory-bound side path, not in the step)
    rope = None
    if not args.no_rope:
        dst = torch.empty_like(path.q)

        def rope_step():
            ops.partition_rope(path.q, w.P, w.layout, 10000.0, ops.ROPE_HALF, out=dst)

        rope_step()
        rms = timed(rope_step, 5, world, flush=flush)
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        moved = 2 * path.q.numel() * path.q.element_size()   # read + write
        rope = {"kernel": "partition_rope_kernel<1>", "ms": rms, "bytes": moved,
                "gbs": moved / (rms * 1e-3) / 1e9, "peak_gbs": hbm,
                "frac_of_hbm": moved / (rms * 1e-3) / 1e9 / hbm, "bound": "hbm",
                "tensor": "q [B, H, N, d] bf16, RoPE split-halves pairs, base 1e4"}
        del dst
        if ops.device_fault():
            raise RuntimeError("device fault during the RoPE partition")

    # ---- CPU oracle baseline (rank 0, one GPU only), and the timed step's
    # output compared with the oracle rows it computes
    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, threads, ref = cpu_oracle_leg(w, 15.0)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc}
        parity = parity_of(o_step, lse_step, v[0, ref[0], 0].double().numpy(), ref)

    peak_key = "bf16_tflops_sustained"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (attn_ms * 1e-3) / 1e12
    traffic = recorded_traffic(w.name)
    # the instance the library launches: work lists for small striped causal
    # problems in the owner schedule (at most 1024 items)
    npairs = -(-(-(-w.c // 128)) // 2)
    lists = (args.sched == "owner" and w.causal and w.layout == W.STRIPED
             and npairs * w.P * w.B * w.H <= 1024)
    kname = (f"attn_fwd_kernel<{w.d}, {'true' if w.layout == W.ZIGZAG else 'false'}, "
             f"{'WorkLists' if lists else 'NoLists'}>")
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peaks_src} {peak_key} (kernel timed inside a seconds-long loop)",
                "frac_of_burst_peak": achieved / burst,
                "frac_of_spec_2250": achieved / SPEC_BF16_TFLOPS,
                "attn_ms_per_launch": attn_ms,
                "attn_ms_median": statistics.median(attn_ts), "attn_ms_min": min(attn_ts),
                "useful_flops_per_launch": flops}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; q,k x3 for the stress workload)",
        "config": config,
        "tokens_per_s": tokens_s,
        "frac_of_peak": value / world / peak,
        "gpu_launches": path.launches_per_step * args.steps,
        "clocks": clocks,
        "roofline": roofline,
        "parity": parity,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "layout_compare": compare,
        "token_order_step": fused,
        "backward": backward,
        "configs": configs,
        "rope_partition": rope,
        "ring_emulation": ring,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
