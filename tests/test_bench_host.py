"""Host-side helpers of bench.py (no GPU): the staleness check of recorded
ncu traffic ignores comments but not code."""

import bench


def test_strip_comments_keeps_code_and_strings():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "// kept";\n'
    assert bench._strip_comments(src) == 'int a = 1; const char* s = "// kept";'


def test_comment_edits_do_not_change_the_code_view():
    a = "x = f(y);  // one reason\n"
    b = "/* another reason */\nx = f(y);\n"
    c = "x = f(z);\n"
    assert bench._strip_comments(a) == bench._strip_comments(b)
    assert bench._strip_comments(a) != bench._strip_comments(c)


def test_recorded_traffic_is_reported_only_for_the_captured_kernel(monkeypatch):
    """The committed DRAM figure is reported while the forward sources hash to
    the captured build, and reads as unknown (None) once they change."""
    import json
    import os
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "attn_fwd_traffic.json")))
    name = "striped_causal_N262144_H16_d128_P16_qk3x"
    e = rec[name]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: e["kernel_hash"])
    assert bench.recorded_traffic(name) == e["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic(name) is None


def _run_bench(args, env_extra=None, timeout=300):
    import os
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py")] + args,
                          capture_output=True, text=True, timeout=timeout, env=env,
                          cwd=bench.ROOT)


def test_reference_arm_prints_one_contract_line():
    import json
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-budget",
                    "0.2", "--workload", "striped_causal_N8192_H16_d128_P8"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["steps"] == 2 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "striped_causal_N8192_H16_d128_P8"
    # the same config object as the GPU arm's line, and the extrapolation named
    assert line["config"] == bench.config_of(
        __import__("long_context_exact_attn_b200.workloads", fromlist=["W"]).BY_NAME[
            "striped_causal_N8192_H16_d128_P8"], "owner", 1)
    assert line["ms_per_step_kind"] == "extrapolated_from_rows"
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # ms_per_step is the whole workload's useful work at the measured rate
    from long_context_exact_attn_b200 import workloads as W
    w = W.BY_NAME["striped_causal_N8192_H16_d128_P8"]
    assert abs(line["ms_per_step"] - w.useful_flops() / (line["value"] * 1e12) * 1e3) < 1e-6 * \
        line["ms_per_step"]


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-budget",
                    "0.1", "--workload", "tiny_noncausal_N256_d64_P4"],
                   env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0


def test_structured_rows_cover_row0_and_shard_edges():
    from long_context_exact_attn_b200 import workloads as W
    w = W.STRIPED_8K
    rows = bench.structured_rows(w)
    assert rows[0] == 0 and w.N - 1 in rows
    # striped: shard j's first local row is token j, its last is (c-1)P + j
    for j in range(w.P):
        assert j in rows and (w.c - 1) * w.P + j in rows
    assert all(0 <= r < w.N for r in rows)


def test_parity_of_reports_errors_against_given_rows():
    import numpy as np
    import torch
    o = torch.zeros(1, 2, 8, 4, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 8)
    o[0, 1, 3] = 0.5
    ref = (1, [0, 3], np.zeros((2, 4)), np.array([0.0, 1e-4]))
    p = bench.parity_of(o, lse, np.zeros(4), ref)
    assert p["rows"] == 2 and p["head"] == 1
    assert p["o_max_abs"] == 0.5 and abs(p["lse_max_abs"] - 1e-4) < 1e-12
    assert p["within"] is False and p["row0_equals_v0"] is True
