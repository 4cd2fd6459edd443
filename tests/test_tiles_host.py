"""The attention kernels' tile classifier, compiled for the host, against the
oracle (no GPU needed).

`csrc/ra_tiles.cuh` holds the integer logic every attention launch uses to
skip, fully compute or mask a 128 x 128 tile (block masks from GetMask,
per-tile thresholds, per-row limits, zigzag chunk masks).  It compiles as
plain C++; `tests/tiles_host.cpp` turns its decisions into a visibility
matrix per (query shard, round) and the tile counts.  Both must equal, bit
for bit, what the oracle derives from the original token positions (the
causal matrix C of the Striped review, 核心公式) and its brute-force tile
census, including ragged shards and tiles cut by the end of a block.
"""

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import masks, work
from oracle.partition import CONTIGUOUS, STRIPED, ZIGZAG

HERE = os.path.dirname(os.path.abspath(__file__))
CODE = {CONTIGUOUS: 0, STRIPED: 1, ZIGZAG: 2}
TILE = 128


@pytest.fixture(scope="module")
def tiles_exe(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler")
    exe = str(tmp_path_factory.mktemp("tiles") / "tiles_host")
    r = subprocess.run([gxx, "-std=c++17", "-O2", "-Wall", "-Wextra", "-Werror",
                        os.path.join(HERE, "tiles_host.cpp"), "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def kernel_view(exe, c, P, layout, causal):
    out = subprocess.run([exe, str(c), str(P), str(CODE[layout]), str(int(causal))],
                         capture_output=True, check=True).stdout
    per = 24 + c * c
    assert len(out) == P * P * per
    res = {}
    for i in range(P * P):
        chunk = out[i * per:(i + 1) * per]
        counts = tuple(int(x) for x in np.frombuffer(chunk[:24], dtype="<i8"))
        vis = np.frombuffer(chunk[24:], dtype=np.uint8).reshape(c, c).astype(bool)
        res[divmod(i, P)] = (counts, vis)
    return res


CASES = [(1, 3), (7, 2), (127, 2), (128, 3), (129, 2), (200, 3), (256, 2), (300, 5), (513, 2)]


@pytest.mark.parametrize("layout", [CONTIGUOUS, STRIPED])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("c,P", CASES)
def test_tile_decisions_equal_positions(tiles_exe, layout, causal, c, P):
    N = c * P
    view = kernel_view(tiles_exe, c, P, layout, causal)
    for (j, r), (counts, vis) in view.items():
        kb = work.key_block(j, r, P)
        blocked = masks.mask_from_positions(j, kb, N, P, layout, causal)
        assert np.array_equal(vis, ~blocked), (j, r)
        skip, full, part, pairs = work.tile_census_brute_force(j, r, N, P, layout, causal,
                                                               TILE, TILE)
        assert counts == (skip, full, part), (j, r)
        assert int(vis.sum()) == pairs


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("c,P", [(512, 1), (512, 2), (512, 3), (1024, 2)])
def test_zigzag_chunk_decisions_equal_positions(tiles_exe, causal, c, P):
    N = c * P
    view = kernel_view(tiles_exe, c, P, ZIGZAG, causal)
    total = 0
    for (j, r), (counts, vis) in view.items():
        kb = work.key_block(j, r, P)
        blocked = masks.mask_from_positions(j, kb, N, P, ZIGZAG, causal)
        assert np.array_equal(vis, ~blocked), (j, r)
        skip, full, part, pairs = work.tile_census_brute_force(j, r, N, P, ZIGZAG, causal,
                                                               TILE, TILE)
        assert counts == (skip, full, part), (j, r)
        total += pairs
    assert total == (N * (N + 1) // 2 if causal else N * N)


def test_a_planted_classifier_error_is_caught(tiles_exe, tmp_path):
    """The comparison is sharp: a copy of the classifier whose striped
    blocks use the strict diagonal everywhere (kb <= j treated like kb > j)
    fails it."""
    src = open(os.path.join(HERE, "..", "long_context_exact_attn_b200", "csrc",
                            "ra_tiles.cuh")).read()
    planted = src.replace("m.e = (kb <= j) ? 1 : 0;", "m.e = 0;")
    assert planted != src
    (tmp_path / "csrc").mkdir()
    (tmp_path / "csrc" / "ra_tiles.cuh").write_text(planted)
    cpp = open(os.path.join(HERE, "tiles_host.cpp")).read().replace(
        '#include "../long_context_exact_attn_b200/csrc/ra_tiles.cuh"', '#include "csrc/ra_tiles.cuh"')
    (tmp_path / "t.cpp").write_text(cpp)
    exe = str(tmp_path / "t")
    subprocess.run([shutil.which("g++"), "-std=c++17", "-O2", "-I", str(tmp_path),
                    str(tmp_path / "t.cpp"), "-o", exe], check=True)
    view = kernel_view(exe, 129, 2, STRIPED, True)
    bad = [(j, r) for (j, r), (_, vis) in view.items()
           if not np.array_equal(vis, ~masks.mask_from_positions(j, work.key_block(j, r, 2),
                                                                 258, 2, STRIPED, True))]
    assert bad
