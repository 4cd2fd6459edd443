"""The profiling build's phase counters (RA_PROFILE, ra_fwd_phase_profile):
run in a separate process (it loads libringattn_prof.so instead of the
regular library), they must count exactly the tiles the kernel computes --
4 softmax warps per (query tile, key tile) pair that is not skipped, from
the oracle's tile census -- and give every phase a plausible cycle count."""

import json
import os
import subprocess
import sys

import pytest
import torch

from long_context_exact_attn_b200 import workloads as W
from oracle import partition as OP
from oracle import work as OW

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("name", ["striped_causal_N8192_H16_d128_P8", "ring_causal_N8192_H16_d128_P8"])
def test_phase_counters_count_the_computed_tiles(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.BY_NAME[name]
    launches = 2
    res = subprocess.run([sys.executable, "-m", "long_context_exact_attn_b200.phase_profile",
                          "--workload", name, "--launches", str(launches)],
                         cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-2000:]
    out = json.loads(res.stdout)
    layout = OP.STRIPED if w.layout == W.STRIPED else OP.CONTIGUOUS
    c = w.N // w.P
    computed = 0
    for j in range(w.P):
        for r in range(w.P):
            _, full, partial = OW.tile_census_closed_form(j, r, c, w.P, layout, w.causal, 128)
            computed += full + partial
    assert out["softmax_tiles"] == launches * 4 * w.B * w.H * computed
    assert out["mma_steps"] > 0
    per_tile = out["softmax_cycles_per_tile"]
    assert all(v >= 0 for v in per_tile.values())
    assert 500 < sum(per_tile.values()) < 200000
    assert all(v >= 0 for v in out["mma_cycles_per_step"].values())
